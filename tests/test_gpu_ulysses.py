"""GPU checks of sequence-parallel (Ulysses) BSA.

1. All R ranks' shards on one GPU in one process (the ranks run one after another): the
   sharded prologue, routing, attention and the inverse relayout into the frame shards give
   O bit for bit equal to the single-GPU pipeline, and so do dq, dk, dv from the sharded
   backward; the gains' gradients, summed over the ranks, agree to fp32 rounding.  The
   single-GPU pipeline is itself checked against the oracle by the other GPU tests, and here
   once more on its attention output.
2. Two processes sharing the GPU, each holding its own frame shards and mapping the other's
   through CUDA IPC (handles exchanged over gloo; the ranks meet only at host barriers, no
   kernel waits for another): each rank's O shard equals the single-GPU result.
"""
import datetime
import os
import socket

import numpy as np
import pytest

from synth import WORKLOADS, Workload, make_raster_inputs
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu


def reference(w, x):
    """Single-GPU pipeline: raster O and input gradients (bf16), dgamma."""
    import torch
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.pipeline import BsaPipeline
    g = bsa.Geometry.from_workload(w)
    pipe = BsaPipeline(g, w.top_r, rope_theta=w.theta, qknorm=True, eps=w.eps, with_bwd=True)
    pipe.set_gamma(to_dev(x["gamma_q"]), to_dev(x["gamma_k"]))
    q, k, v, do = (to_dev(x[n]) for n in ("q", "k", "v", "do"))
    pipe.forward(q, k, v)
    pipe.load_grad(do)
    pipe.backward()
    o = torch.empty_like(q)
    one = bsa.Shards(1, w.t_frames, w.heads, 0)
    bsa.bsa_blocked_to_raster_sharded(g, w.t_frames, one, pipe.o, [o])
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    dgq = torch.empty(w.head_dim, device="cuda")
    dgk = torch.empty_like(dgq)
    pipe.prologue_backward(q, k, dq, dk, dv, dgq, dgk)
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == 0
    return pipe, {"o": o, "dq": dq, "dk": dk, "dv": dv, "dgq": dgq, "dgk": dgk}


def frame_shards(t, world, tokens_per_shard):
    return [t[:, s * tokens_per_shard:(s + 1) * tokens_per_shard].contiguous() for s in range(world)]


@pytest.mark.parametrize("name,world", [("small", 2), ("small_b2", 3), ("ulysses_8", 8)])
def test_sharded_ranks_in_one_process_match_single_gpu(name, world):
    import torch
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.ulysses import UlyssesBsa, UlyssesPlan
    from tests.test_gpu_fwd import check_attention
    w = WORKLOADS.get(name) or Workload("ulysses_8", 1, 16, 128, 16, 12, 20, (4, 4, 8), 6,
                                         unit_gamma=False)
    x = make_raster_inputs(w, with_grad=True)
    pipe, ref = reference(w, x)
    check_attention(w, pipe, [0, w.heads - 1])
    g = bsa.Geometry.from_workload(w)
    F = w.t_frames // world
    tps = F * w.grid_h * w.grid_w
    sh = {n: frame_shards(to_dev(x[n]), world, tps) for n in ("q", "k", "v", "do")}
    for n in ("o", "dq", "dk", "dv"):
        sh[n] = [torch.zeros_like(t) for t in sh["q"]]
    ptrs = {n: [t.data_ptr() for t in ts] for n, ts in sh.items()}
    gq, gk = to_dev(x["gamma_q"]), to_dev(x["gamma_k"])
    ranks = [UlyssesBsa(UlyssesPlan(world, r, w.heads, w.t_frames), g, w.top_r, ptrs,
                        rope_theta=w.theta, gamma_q=gq, gamma_k=gk, eps=w.eps, with_bwd=True)
             for r in range(world)]
    for u in ranks:
        u.forward()
    torch.cuda.synchronize()  # every O shard written (the barrier of the multi-GPU case)
    for u in ranks:
        u.backward()
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == 0
    for n in ("o", "dq", "dk", "dv"):
        got = torch.cat(sh[n], dim=1)
        assert torch.equal(got.view(torch.int16), ref[n].view(torch.int16)), n
    for n, attr in (("dgq", "dgamma_q"), ("dgk", "dgamma_k")):
        tot = sum(getattr(u, attr) for u in ranks)
        err = (tot - ref[n]).abs().max().item()
        assert err <= 1e-5 * ref[n].abs().max().item() + 1e-6, (n, err)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _ipc_rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=90))
    opened = []
    try:
        import block_sparse_attention_route_b200 as bsa
        from block_sparse_attention_route_b200.ulysses import (UlyssesBsa, UlyssesPlan,
                                                               close_pointers, exchange_pointers,
                                                               rank_barrier)
        torch.cuda.set_device(0)
        w = WORKLOADS["small"]
        x = make_raster_inputs(w, with_grad=True)
        _, ref = reference(w, x)
        plan = UlyssesPlan(world, rank, w.heads, w.t_frames)
        tps = plan.shard_tokens(bsa.Geometry.from_workload(w))
        mine = {n: frame_shards(to_dev(x[n]), world, tps)[rank] for n in ("q", "k", "v")}
        mine["o"] = torch.zeros_like(mine["q"])
        table, opened = exchange_pointers(mine)
        u = UlyssesBsa(plan, bsa.Geometry.from_workload(w), w.top_r, table, rope_theta=w.theta,
                       gamma_q=to_dev(x["gamma_q"]), gamma_k=to_dev(x["gamma_k"]), eps=w.eps)
        rank_barrier()  # every rank's q, k, v shard is in place
        u.forward()
        rank_barrier()  # every rank has written its heads into every O shard
        assert bsa.bsa_device_status() == 0
        exp = ref["o"][:, rank * tps:(rank + 1) * tps]
        ok = torch.equal(mine["o"].view(torch.int16), exp.view(torch.int16))
        rank_barrier()  # no rank unmaps while another still writes
        close_pointers(opened)
        opened = []
        q.put((rank, "ok" if ok else "O shard differs"))
    except Exception as e:  # report instead of leaving the other rank at a barrier
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


def test_two_processes_share_shards_through_ipc():
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ipc_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=240) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    assert res == [(r, "ok") for r in range(world)], res
