"""Host logic of sequence-parallel (Ulysses) BSA, on CPU with gloo ranks.

The plan (which rank holds which frames and computes which heads), the exchange of shard
pointers between ranks (with a stand-in for CUDA IPC), and the index map the sharded kernels
use to read a (frame, head) row from the frame shards, checked against a real all-to-all
between gloo ranks.
"""
import os
import socket
import struct

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_route_b200.ulysses import UlyssesPlan, exchange_pointers


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_plan_splits_frames_and_heads():
    for world in (1, 2, 3, 4, 6, 8):
        plans = [UlyssesPlan(world, r, 48, 24) for r in range(world)]
        assert [p.head0 for p in plans] == [r * 48 // world for r in range(world)]
        assert all(p.heads_local * world == 48 and p.shard_frames * world == 24 for p in plans)
        assert plans[-1].frame0 + plans[-1].shard_frames == 24
        sh = plans[-1].shards()
        assert (sh.n_shards, sh.shard_frames, sh.heads_total, sh.head0) == (world, 24 // world, 48,
                                                                             plans[-1].head0)
    for bad in (dict(world=5), dict(world=9), dict(rank=2, world=2)):
        args = dict(world=2, rank=0, heads=48, frames=24)
        args.update(bad)
        with pytest.raises(ValueError):
            UlyssesPlan(**args)


def _shard_row(shards, F, tokens_per_frame, t, n_in_frame, h):
    """The sharded kernels' index map: frame t lives in shard t // F at local token
    (t - s F) * tokens_per_frame + n_in_frame; rows keep all heads."""
    s = t // F
    return shards[s][:, (t - s * F) * tokens_per_frame + n_in_frame, h]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # ---- pointer exchange with a stand-in for CUDA IPC
        def fake_export(t):
            return struct.pack("<qq", rank, t.data_ptr()).ljust(128, b"\0")

        def fake_import(h):
            r, p = struct.unpack("<qq", h[:16])
            return (r + 1) << 48 | (p & 0xFFFFFFFFFFFF)

        mine = {"q": torch.zeros(8), "o": torch.zeros(4)}
        table, opened = exchange_pointers(mine, export=fake_export, import_=fake_import)
        for n in ("q", "o"):
            assert len(table[n]) == world
            for r, p in enumerate(table[n]):
                if r == rank:
                    assert p == mine[n].data_ptr()
                else:
                    assert p >> 48 == r + 1
        assert len(opened) == 2 * (world - 1)

        # ---- the sharded index map against a real all-to-all (sequence -> head)
        B, T, HW, H, D = 1, 6, 5, 6, 3
        plan = UlyssesPlan(world, rank, H, T)
        F, Hl = plan.shard_frames, plan.heads_local
        rng = np.random.default_rng(0)
        full = torch.from_numpy(rng.standard_normal((B, T * HW, H, D)).astype(np.float32))
        mine = full[:, plan.frame0 * HW:(plan.frame0 + F) * HW].contiguous()  # my frames
        # all-to-all: send to rank s my frames of its heads, receive my heads of everyone's frames
        send = torch.cat([mine[:, :, s * Hl:(s + 1) * Hl].reshape(-1) for s in range(world)])
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send)
        got = recv.view(world, B, F * HW, Hl, D).permute(1, 0, 2, 3, 4).reshape(B, T * HW, Hl, D)
        assert torch.equal(got, full[:, :, plan.head0:plan.head0 + Hl])
        # the pointer-table view: every rank's shard, indexed the way the kernels do
        shards = [full[:, s * F * HW:(s + 1) * F * HW] for s in range(world)]
        for t in range(T):
            for n in range(HW):
                for h in range(Hl):
                    assert torch.equal(_shard_row(shards, F, HW, t, n, plan.head0 + h), got[:, t * HW + n, h])

        # ---- head -> sequence for O: the inverse all-to-all gives my frames of all heads
        o_local = got * 2.0 + rank  # stand-in for this rank's attention output (its heads)
        send = torch.cat([o_local[:, s * F * HW:(s + 1) * F * HW].reshape(-1) for s in range(world)])
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send)
        o_mine = recv.view(world, B, F * HW, Hl, D).permute(1, 2, 0, 3, 4).reshape(B, F * HW, H, D)
        expect = torch.cat([full[:, plan.frame0 * HW:(plan.frame0 + F) * HW, r * Hl:(r + 1) * Hl] * 2.0 + r
                            for r in range(world)], dim=2)
        assert torch.equal(o_mine, expect)
        q.put((rank, "ok"))
    except Exception as e:  # report to the parent instead of hanging the group
        q.put((rank, repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_exchange_and_index_map_match_all_to_all(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
    assert sorted(res) == [(r, "ok") for r in range(world)], res


def test_rank_runner_rejects_inconsistent_setups_before_allocating():
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.ulysses import UlyssesBsa
    g = bsa.Geometry(1, 32, 128, 24, 45, 80)
    with pytest.raises(ValueError):  # a continuation cache is not sequence-parallel here
        UlyssesBsa(UlyssesPlan(8, 0, 32, 24), bsa.Geometry(1, 32, 128, 24, 45, 80, cached_t=4), 72, {})
    with pytest.raises(ValueError):  # plan for other heads than the geometry's
        UlyssesBsa(UlyssesPlan(8, 0, 16, 24), g, 72, {})
    with pytest.raises(ValueError):  # plan for other frames
        UlyssesBsa(UlyssesPlan(8, 0, 32, 16), g, 72, {})
    gl = UlyssesPlan(8, 3, 32, 24).local_geometry(g)
    assert (gl.heads, gl.t_frames, gl.grid_h) == (4, 24, 45)
