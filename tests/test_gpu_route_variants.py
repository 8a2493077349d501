"""GPU parity of the routing variants (bsa_route_ex flags) against the oracle's route.

The oracle is fed the GPU's bf16 post-prologue q / k (and cached keys), as in the plain
routing tests; selections must match exactly except for near ties (within 1e-4 relative of
the threshold score).  With the forced self-block the own block must be present and the
near-tie rule applies to the other r - 1 places; with head-shared routing every head's row
must be the same selection, ranked by the score summed over heads.  Attention then runs on
a variant's selection and is compared with the oracle's attention on those blocks.
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOADS
from tests.helpers import grid_of
from tests.test_gpu_fwd import check_attention, head_raster, run_forward

pytestmark = pytest.mark.gpu

FS, SH, PSUM, PMAX = 1, 2, 4, 8
VARIANTS = {"force_self": FS, "shared_heads": SH, "self_shared": FS | SH, "pool_sum": PSUM,
            "pool_max": PMAX, "max_self_shared": PMAX | FS | SH}


def oracle_route(w, pipe, flags, heads):
    """Oracle route of the given heads (all heads when shared) on the GPU's q / k."""
    grid = grid_of(w)
    sm = grid.slot_map(w.t_frames)
    pool = "sum" if flags & PSUM else "max" if flags & PMAX else "mean"
    hs = list(range(w.heads)) if flags & SH else heads
    q = np.concatenate([head_raster(pipe.q, sm, h) for h in hs], axis=2)
    k = np.concatenate([head_raster(pipe.k, sm, h) for h in hs], axis=2)
    kc = None
    if w.cached_t:
        smc = grid.slot_map(w.cached_t)
        kc = np.concatenate([head_raster(pipe.kc, smc, h) for h in hs], axis=2)
    return oracle.route(q, k, grid, pipe.r, k_cache=kc, pool=pool, force_self=bool(flags & FS),
                        shared_heads=bool(flags & SH))


def compare(w, pipe, flags, heads, ridx, rcnt, s, rows=None):
    grid = grid_of(w)
    idx = pipe.idx.cpu().numpy()
    cnt = pipe.cnt.cpu().numpy()
    exempt = 0
    for b in range(w.batch):
        for n, h in enumerate(heads):
            o = 0 if flags & SH else n
            for i in (rows if rows is not None else range(grid.nbq)):
                gsel, osel = idx[b, h, i], ridx[b, o if not flags & SH else h, i]
                assert cnt[b, h, i] == rcnt[b, o if not flags & SH else h, i], (b, h, i)
                assert np.all(gsel[cnt[b, h, i]:] == -1)
                if flags & FS:
                    assert grid.nbc + i in gsel
                if flags & SH:
                    assert np.array_equal(gsel, idx[b, 0, i])
                if np.array_equal(gsel, osel):
                    continue
                assert np.all(np.diff(gsel[:cnt[b, h, i]]) > 0)
                own = {grid.nbc + i} if flags & FS else set()
                g_o = [j for j in gsel if j not in own]
                o_o = [j for j in osel if j not in own]
                assert oracle.near_tie_ok(g_o, o_o, s[b, 0 if flags & SH else o, i]), (b, h, i, gsel, osel)
                exempt += 1
    return exempt


@pytest.mark.parametrize("name", ["small", "small_b2", "small_cont", "tiny_ragged"])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_route_variant_parity_small(name, variant):
    w = WORKLOADS[name]
    flags = VARIANTS[variant]
    pipe, _ = run_forward(w)
    pipe.route(flags=flags)
    pipe.attn_fwd()
    heads = list(range(w.heads))
    ridx, rcnt, s = oracle_route(w, pipe, flags, heads)
    assert compare(w, pipe, flags, heads, ridx, rcnt, s) == 0
    check_attention(w, pipe, heads)


def test_force_self_r1_attends_only_to_the_own_block():
    w = WORKLOADS["small_cont"]
    pipe, _ = run_forward(w, top_r=1)
    pipe.route(flags=FS)
    pipe.attn_fwd()
    g = grid_of(w)
    idx = pipe.idx.cpu().numpy()
    assert np.array_equal(idx[..., 0], np.broadcast_to(g.nbc + np.arange(g.nbq), idx.shape[:3]))
    check_attention(w, pipe, list(range(w.heads)))


@pytest.mark.parametrize("variant", ["force_self", "shared_heads"])
def test_route_variant_720p_sampled(variant):
    """The measured 720p geometry, in the launch configuration the bench times; the shared
    selection is checked on sampled rows with scores summed over all 32 heads."""
    w = WORKLOADS["720p"]
    flags = VARIANTS[variant]
    pipe, _ = run_forward(w)
    pipe.route(flags=flags)
    grid = grid_of(w)
    rng = np.random.default_rng(7)
    rows = sorted(set(int(i) for i in rng.integers(0, grid.nbq, 40)) | {0, grid.nbq - 1})
    heads = [0, 21]
    if flags & SH:
        # sum the oracle's per-head scores head by head (keeps host memory small)
        sm = grid.slot_map(w.t_frames)
        mem = grid.block_members(w.t_frames)
        s = 0.0
        for h in range(w.heads):
            qb = oracle.block_pool(head_raster(pipe.q, sm, h), mem)
            kb = oracle.block_pool(head_raster(pipe.k, sm, h), mem)
            s = s + oracle.block_scores(qb[:, :, rows], kb, grid)
        ridx, rcnt = oracle.select_top_r(s, pipe.r)
        ridx = np.repeat(ridx, w.heads, axis=1)
        rcnt = np.repeat(rcnt, w.heads, axis=1)
        sfull = s
        # compare() indexes rows by query block: expand to full row arrays
        full_idx = -np.ones((1, w.heads, grid.nbq, pipe.r), dtype=np.int32)
        full_cnt = np.zeros((1, w.heads, grid.nbq), dtype=np.int32)
        full_s = np.zeros((1, 1, grid.nbq, grid.nbk))
        full_idx[:, :, rows], full_cnt[:, :, rows], full_s[:, :, rows] = ridx, rcnt, sfull
        exempt = compare(w, pipe, flags, heads, full_idx, full_cnt, full_s, rows)
    else:
        ridx, rcnt, s = oracle_route(w, pipe, flags, heads)
        exempt = compare(w, pipe, flags, heads, ridx, rcnt, s, rows)
    assert exempt <= 1


@pytest.mark.parametrize("variant", ["plain", "self_shared"])
def test_route_at_the_key_block_limit(variant):
    """4096 key blocks per head (the library's limit): the score rows fill most of the
    select kernel's shared memory (8 query rows per CTA); sampled rows against the oracle."""
    from synth import Workload
    from tests.test_gpu_fwd import check_route
    w = Workload("max_blocks", 1, 2, 128, 128, 64, 64, (4, 4, 8), 8, rope=False, qknorm=False)
    grid = grid_of(w)
    assert grid.nbk == 4096
    pipe, _ = run_forward(w)
    rng = np.random.default_rng(11)
    rows = sorted(set(int(i) for i in rng.integers(0, grid.nbq, 24)) | {0, grid.nbq - 1})
    if variant == "plain":
        assert check_route(w, pipe, [0, 1], rows) <= 1
        check_attention(w, pipe, [1], qblocks=rows[:6])
    else:
        flags = VARIANTS[variant]
        pipe.route(flags=flags)
        ridx, rcnt, s = oracle_route(w, pipe, flags, [0, 1])
        assert compare(w, pipe, flags, [0, 1], ridx, rcnt, s, rows) <= 1
