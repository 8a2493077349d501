"""Head sharding over 2 ranks (gloo, CPU): each rank computes its head slice of the BSA
forward (oracle, since this runs without a GPU) and the all-gather over heads reproduces the
single-process result exactly."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_route_b200.shard import head_range


def test_head_range_partitions():
    for heads in (1, 2, 3, 7, 32):
        for world in (1, 2, 3, 4, 8):
            rs = [head_range(r, world, heads) for r in range(world)]
            assert rs[0][0] == 0 and rs[-1][1] == heads
            assert all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
            assert max(h1 - h0 for h0, h1 in rs) - min(h1 - h0 for h0, h1 in rs) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from block_sparse_attention_route_b200.shard import gather_heads
        from synth import WORKLOADS, bf16_bits_to_f64, make_raster_inputs
        w = WORKLOADS["small_b2"]  # 3 heads over 2 ranks: uneven split
        x = make_raster_inputs(w)
        h0, h1 = head_range(rank, world, w.heads)
        grid = oracle.Grid(w.t_frames, w.grid_h, w.grid_w, w.blk)
        q = oracle.prologue(bf16_bits_to_f64(x["q"])[:, :, h0:h1], w.t_frames, w.grid_h, w.grid_w,
                            gamma=x["gamma_q"], theta=w.theta)
        k = oracle.prologue(bf16_bits_to_f64(x["k"])[:, :, h0:h1], w.t_frames, w.grid_h, w.grid_w,
                            gamma=x["gamma_k"], theta=w.theta)
        v = bf16_bits_to_f64(x["v"])[:, :, h0:h1]
        idx, _, _ = oracle.route(q, k, grid, w.top_r)
        o, _ = oracle.attend(q, k, v, idx, grid, 1.0 / math.sqrt(w.head_dim))
        full = gather_heads(torch.from_numpy(o), w.heads, dim=2)
        if rank == 0:
            out.put(full.numpy())
    finally:
        dist.destroy_process_group()


def test_gather_heads_two_ranks_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from synth import WORKLOADS, bf16_bits_to_f64, make_raster_inputs
    w = WORKLOADS["small_b2"]
    x = make_raster_inputs(w)
    grid = oracle.Grid(w.t_frames, w.grid_h, w.grid_w, w.blk)
    qf = oracle.prologue(bf16_bits_to_f64(x["q"]), w.t_frames, w.grid_h, w.grid_w,
                         gamma=x["gamma_q"], theta=w.theta)
    kf = oracle.prologue(bf16_bits_to_f64(x["k"]), w.t_frames, w.grid_h, w.grid_w,
                         gamma=x["gamma_k"], theta=w.theta)
    idx, _, _ = oracle.route(qf, kf, grid, w.top_r)
    of, _ = oracle.attend(qf, kf, bf16_bits_to_f64(x["v"]), idx, grid, 1.0 / math.sqrt(w.head_dim))
    np.testing.assert_array_equal(got, of)
