"""Pins for the fp64 oracle against facts it does not compute itself.

Each test fixes the oracle to something independent of its own code: a textbook or library
routine (torch CPU scaled_dot_product_attention and autograd in fp64), a pure-Python brute
force on tiny grids, closed forms of the rotary embedding, invariants of softmax and RoPE,
or numerical derivatives.  None of these needs a GPU.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from oracle import Grid
from synth import WORKLOADS, bf16_bits_to_f64, make_raster_inputs

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _grid(w):
    return Grid(w.t_frames, w.grid_h, w.grid_w, w.blk, w.cached_t, w.chunk_t, w.cond_t)


def _inputs(name):
    w = WORKLOADS[name]
    x = make_raster_inputs(w, with_grad=True)
    return w, {k: (bf16_bits_to_f64(v) if v is not None and v.dtype == np.uint16 else v)
               for k, v in x.items()}


def _sdpa(q, k, v, scale, mask=None, need_grad=False):
    """torch CPU fp64 SDPA on raster [B, N, H, D] arrays; mask [B, H, N, Nk] bool (True = keep)."""
    tq, tk, tv = (torch.tensor(a.transpose(0, 2, 1, 3).copy(), dtype=torch.float64,
                               requires_grad=need_grad) for a in (q, k, v))
    m = None if mask is None else torch.tensor(mask)
    o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=m, scale=scale)
    return o, (tq, tk, tv)


# ------------------------------------------------------------------ layout / geometry
def test_slot_map_matches_block_members():
    for name in ("tiny", "tiny_ragged", "small", "small_b2"):
        g = _grid(WORKLOADS[name])
        sm = g.slot_map(g.t_frames)
        mem = g.block_members(g.t_frames)
        for b in range(g.nbq):
            valid = [int(x) for x in sm[b] if x >= 0]
            assert valid == mem[b]
        # every token appears exactly once
        allv = np.sort(sm[sm >= 0])
        assert np.array_equal(allv, np.arange(g.t_frames * g.grid_h * g.grid_w))


def test_block_numbering_worked_by_hand():
    """Tokens of a ragged 5 x 6 x 10 grid (t, h, w) cut into 4 x 4 x 8 blocks, worked by hand.

    Blocks per axis: ceil(5/4) = 2, ceil(6/4) = 2, ceil(10/8) = 2, numbered
    (block-t * 2 + block-h) * 2 + block-w.  Raster index of a token = (t * 6 + h) * 10 + w.
    Valid extents (vt, vh, vw) per block (the last block along an axis keeps 1 frame, 2 rows
    or 2 columns) and valid tokens: block 0 (4,4,8) 128, 1 (4,4,2) 32, 2 (4,2,8) 64,
    3 (4,2,2) 16, 4 (1,4,8) 32, 5 (1,4,2) 8, 6 (1,2,8) 16, 7 (1,2,2) 4.
    Slot inside a block = (local t * vh + local h) * vw + local w (pad slots after them):
      (t, h, w) = (0, 0, 0): raster 0,   block 0, local (0, 0, 0), slot 0
      (1, 2, 3):             raster 83,  block 0, local (1, 2, 3), slot (1*4 + 2)*8 + 3 = 51
      (2, 1, 9):             raster 139, block 1, local (2, 1, 1), slot (2*4 + 1)*2 + 1 = 19
      (3, 4, 8):             raster 228, block 3, local (3, 0, 0), slot (3*2 + 0)*2 + 0 = 12
      (4, 0, 2):             raster 242, block 4, local (0, 0, 2), slot 2
      (4, 5, 9):             raster 299, block 7, local (0, 1, 1), slot (0*2 + 1)*2 + 1 = 3
    The block grid is a 2 x 2 x 2 cube, so only the order of the axes tells these ids apart.
    """
    g = Grid(5, 6, 10, (4, 4, 8))
    sm = g.slot_map(5)
    mem = g.block_members(5)
    for (t, h, w), (raster, blk, slot) in {(0, 0, 0): (0, 0, 0), (1, 2, 3): (83, 0, 51),
                                           (2, 1, 9): (139, 1, 19), (3, 4, 8): (228, 3, 12),
                                           (4, 0, 2): (242, 4, 2), (4, 5, 9): (299, 7, 3)}.items():
        assert (t * 6 + h) * 10 + w == raster
        assert sm[blk, slot] == raster
        assert raster in mem[blk]
    assert [len(m) for m in mem] == [128, 32, 64, 16, 32, 8, 16, 4]
    assert mem[7] == [280 + 8, 280 + 9, 290 + 8, 290 + 9]  # (4,4,8) (4,4,9) (4,5,8) (4,5,9)
    assert sm[7].tolist() == [288, 289, 298, 299] + [-1] * 124  # valid prefix, then pads
    assert [int((row >= 0).sum()) for row in sm] == [128, 32, 64, 16, 32, 8, 16, 4]
    assert all(np.all(row[:n] >= 0) and np.all(row[n:] < 0)
               for row, n in zip(sm, [128, 32, 64, 16, 32, 8, 16, 4]))


def test_workload_geometry_matches_pages():
    """Golden geometry: latent grid and block counts of the measured workloads."""
    import json
    import os
    with open(os.path.join(os.path.dirname(__file__), "golden", "geometry.json")) as f:
        gold = json.load(f)
    for name, rec in gold["workloads"].items():
        w = WORKLOADS[name]
        assert [w.t_frames + w.cached_t, w.grid_h, w.grid_w] == rec["latent_grid"]
        nbq, nbc = w.n_blocks()
        assert nbq + nbc == rec["key_blocks"]
        assert nbq == rec["query_blocks"]
        assert w.top_r == rec["top_r"]
        assert abs(w.top_r / (nbq + nbc) - rec["density"]) < 5e-3


# ------------------------------------------------------------------ prologue pins
def test_rope_closed_form_small_head():
    """D = 12: split (4, 4, 4), theta = 10000.  Hand-worked angles at position (1, 2, 3):
    t pairs turn by 1 and 0.01 rad, h pairs by 2 and 0.02, w pairs by 3 and 0.03."""
    assert oracle.rope_split(12) == (4, 4, 4)
    x = np.zeros((1, 1, 1, 12))
    x[..., 0::2] = 1.0  # every pair = (1, 0)
    y = oracle.rope3d(x, np.array([1.0]), np.array([2.0]), np.array([3.0]), 10000.0)
    angles = [1.0, 0.01, 2.0, 0.02, 3.0, 0.03]
    for p, a in enumerate(angles):
        assert y[0, 0, 0, 2 * p] == pytest.approx(math.cos(a), abs=1e-15)
        assert y[0, 0, 0, 2 * p + 1] == pytest.approx(math.sin(a), abs=1e-15)


def test_rope_split_head128():
    assert oracle.rope_split(128) == (44, 42, 42)
    assert oracle.rope_split(64) == (24, 20, 20)


def test_rope_position_zero_is_identity_and_norm_preserving():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 6, 3, 128))
    z = np.zeros(6)
    assert np.array_equal(oracle.rope3d(x, z, z, z, 10000.0), x)
    pos = rng.integers(0, 90, size=(3, 6)).astype(np.float64)
    y = oracle.rope3d(x, pos[0], pos[1], pos[2], 10000.0)
    pn_x = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    pn_y = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(pn_y, pn_x, rtol=1e-12, atol=1e-12)


def test_rope_relative_position_per_axis():
    """q(m) . k(n) depends only on m - n along each axis."""
    rng = np.random.default_rng(7)
    q = rng.standard_normal((1, 1, 1, 128))
    k = rng.standard_normal((1, 1, 1, 128))

    def dot(m, n):
        a = oracle.rope3d(q, *[np.array([float(c)]) for c in m], 10000.0)
        b = oracle.rope3d(k, *[np.array([float(c)]) for c in n], 10000.0)
        return float(np.sum(a * b))
    base = dot((5, 7, 11), (2, 3, 4))
    assert dot((3, 4, 7), (0, 0, 0)) == pytest.approx(base, rel=1e-11, abs=1e-11)
    assert dot((20, 30, 40), (17, 26, 33)) == pytest.approx(base, rel=1e-11, abs=1e-11)
    assert dot((5, 7, 11), (2, 3, 5)) != pytest.approx(base, rel=1e-6)


def test_rmsnorm_unit_rms_and_commutes_with_rope():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((1, 10, 2, 128)) * 3.0
    g1 = np.ones(128)
    y = oracle.rms_norm(x, g1, 1e-6)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-6)
    t, h, w = oracle.grid_positions(1, 2, 5, t_offset=3)
    a = oracle.rope3d(oracle.rms_norm(x, g1, 1e-6), t, h, w, 10000.0)
    b = oracle.rms_norm(oracle.rope3d(x, t, h, w, 10000.0), g1, 1e-6)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    # a gain scales channels after normalisation
    gam = rng.standard_normal(128)
    np.testing.assert_allclose(oracle.rms_norm(x, gam, 1e-6), y * gam, rtol=1e-12)


def test_prologue_positions_follow_raster_order():
    """Token n of a (T, Hg, Wg) raster sits at (n // (Hg Wg), (n // Wg) % Hg, n % Wg)."""
    t, h, w = oracle.grid_positions(3, 4, 5, t_offset=2)
    n = np.arange(60)
    assert np.array_equal(t, n // 20 + 2)
    assert np.array_equal(h, (n // 5) % 4)
    assert np.array_equal(w, n % 5)


# ------------------------------------------------------------------ routing pins
def _brute_route(q, k, grid, r):
    """Pure-Python scalar routing on tiny grids (loops only)."""
    B, N, H, D = q.shape
    mem = grid.block_members(grid.t_frames)
    idx_all, cnt_all = {}, {}
    for b in range(B):
        for h in range(H):
            means = []
            for arr in (q, k):
                ms = []
                for toks in mem:
                    ms.append([sum(float(arr[b, t, h, d]) for t in toks) / len(toks)
                               for d in range(D)])
                means.append(ms)
            for i in range(grid.nbq):
                sc = []
                for j in range(grid.nbk):
                    s = sum(means[0][i][d] * means[1][j][d] for d in range(D))
                    if grid.masked and grid.key_block_chunk(j) > grid.query_block_chunk(i):
                        s = -math.inf
                    sc.append(s)
                chosen = []
                left = list(range(grid.nbk))
                while len(chosen) < r:
                    best = None
                    for j in left:
                        if sc[j] == -math.inf:
                            continue
                        if best is None or sc[j] > sc[best]:
                            best = j  # strict '>' keeps the lower index on ties
                    if best is None:
                        break
                    chosen.append(best)
                    left.remove(best)
                idx_all[(b, h, i)] = sorted(chosen)
                cnt_all[(b, h, i)] = len(chosen)
    return idx_all, cnt_all


@pytest.mark.parametrize("name", ["tiny", "tiny_ragged"])
def test_route_brute_force(name):
    w, x = _inputs(name)
    g = _grid(w)
    idx, cnt, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    bi, bc = _brute_route(x["q"], x["k"], g, w.top_r)
    for key, sel in bi.items():
        b, h, i = key
        assert cnt[b, h, i] == bc[key]
        assert list(idx[b, h, i, :cnt[b, h, i]]) == sel
        assert all(v == -1 for v in idx[b, h, i, cnt[b, h, i]:])


def test_route_brute_force_causal():
    g = Grid(8, 4, 4, (2, 4, 4), chunk_t=4)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 128, 1, 8))
    k = rng.standard_normal((1, 128, 1, 8))
    idx, cnt, _ = oracle.route(q, k, g, 3)
    bi, bc = _brute_route(q, k, g, 3)
    for (b, h, i), sel in bi.items():
        assert list(idx[b, h, i, :cnt[b, h, i]]) == sel and cnt[b, h, i] == bc[(b, h, i)]
    # query blocks 0,1 (chunk 0) may only see key blocks 0,1: cnt = 2 < r
    assert list(cnt[0, 0]) == [2, 2, 3, 3]
    assert list(idx[0, 0, 0]) == [0, 1, -1]


def test_route_exact_ties_lower_index_wins():
    g = Grid(2, 4, 16, (2, 4, 4))  # 4 blocks along w
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 128, 1, 16))
    k = rng.standard_normal((1, 128, 1, 16))
    mem = g.block_members(2)
    k[0, mem[3]] = k[0, mem[1]]  # blocks 1 and 3 identical -> equal scores for every query
    _, _, s = oracle.route(q, k, g, 1)
    for i in range(4):
        assert s[0, 0, i, 1] == s[0, 0, i, 3]
    # force blocks 1 and 3 to be the two largest, so r = 1 must pick block 1
    q[0, :] = 0.0
    q[0, mem[0]] = k[0, mem[1]].mean(axis=0)
    idx, cnt, s = oracle.route(q, k, g, 1)
    assert s[0, 0, 0, 1] == s[0, 0, 0, 3]
    assert idx[0, 0, 0, 0] == 1


def test_route_proportional_block_ranks_first():
    g = Grid(4, 8, 8, (2, 4, 4))
    rng = np.random.default_rng(13)
    k = rng.standard_normal((1, 256, 1, 64))
    mem = g.block_members(4)
    kbar5 = k[0, mem[5], 0].mean(axis=0)
    q = rng.standard_normal((1, 256, 1, 64)) * 1e-3
    q[0, mem[2], 0] += 10.0 * kbar5  # query block 2 is aligned with key block 5
    _, _, s = oracle.route(q, k, g, 8)
    assert int(np.argmax(s[0, 0, 2])) == 5


def test_route_all_blocks_when_r_equals_nb():
    w, x = _inputs("tiny")
    g = _grid(w)
    idx, cnt, _ = oracle.route(x["q"], x["k"], g, g.nbk)
    assert np.all(cnt == g.nbk)
    assert np.array_equal(idx[0, 0, 3], np.arange(g.nbk))


def test_route_causal_never_selects_later_chunk():
    w, x = _inputs("small_cont")
    g = _grid(w)
    idx, cnt, s = oracle.route(x["q"], x["k"], g, w.top_r, k_cache=x["kc"])
    for i in range(g.nbq):
        for j in idx[0, 0, i]:
            if j >= 0:
                assert g.key_block_chunk(int(j)) <= g.query_block_chunk(i)
    # continuation: key blocks 0..nbc-1 are cached, all cached chunks precede the queries
    assert g.nbc == g.nbq


def test_near_tie_rule():
    row = np.array([0.5, 0.30000, 0.300001, 0.1, -np.inf])
    assert oracle.near_tie_ok([0, 1], [0, 1], row)
    assert oracle.near_tie_ok([0, 1], [0, 2], row)          # 0.3 vs 0.300001: within 1e-4
    assert not oracle.near_tie_ok([0, 3], [0, 2], row)      # 0.1 is far from tau
    assert not oracle.near_tie_ok([0], [0, 2], row)         # counts differ


# ------------------------------------------------------------------ attention pins
def _token_mask(grid, idx, B, H):
    """Dense token-level keep mask [B, H, N, N] from block selections (current keys only)."""
    mem = grid.block_members(grid.t_frames)
    n = grid.t_frames * grid.grid_h * grid.grid_w
    m = np.zeros((B, H, n, n), dtype=bool)
    for b in range(B):
        for h in range(H):
            for i, qi in enumerate(mem):
                for j in idx[b, h, i]:
                    if j >= 0:
                        m[b, h, np.ix_(qi, mem[j])[0], np.ix_(qi, mem[j])[1]] = True
    return m


@pytest.mark.parametrize("name", ["tiny", "tiny_ragged", "tiny_d128"])
def test_all_blocks_equals_dense_sdpa(name):
    w, x = _inputs(name)
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, _, _ = oracle.route(x["q"], x["k"], g, g.nbk)
    o, lse = oracle.attend(x["q"], x["k"], x["v"], idx, g, scale)
    ref, _ = _sdpa(x["q"], x["k"], x["v"], scale)
    np.testing.assert_allclose(o, ref.detach().numpy().transpose(0, 2, 1, 3), atol=1e-12)
    od, lsed = oracle.dense_attention(x["q"], x["k"], x["v"], scale)
    np.testing.assert_allclose(lse, lsed, atol=1e-12)
    # LSE against a direct log-sum-exp of the logits of one token
    qv, kv = x["q"][0, 17, 1], x["k"][0, :, 1]
    logits = kv @ qv * scale
    assert lse[0, 17, 1] == pytest.approx(math.log(np.sum(np.exp(logits))), rel=1e-12)


@pytest.mark.parametrize("name", ["tiny", "tiny_ragged"])
def test_sparse_equals_masked_sdpa(name):
    """Attention over the selected blocks equals dense attention with every other key masked
    (torch's boolean mask gives masked keys exactly zero weight)."""
    w, x = _inputs(name)
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, _, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    o, _ = oracle.attend(x["q"], x["k"], x["v"], idx, g, scale)
    mask = _token_mask(g, idx, w.batch, w.heads)
    ref, _ = _sdpa(x["q"], x["k"], x["v"], scale, mask=mask)
    np.testing.assert_allclose(o, ref.detach().numpy().transpose(0, 2, 1, 3), atol=1e-12)


def _brute_attend_token(q, k, v, idx_row, grid, b, h, n, scale):
    mem = grid.block_members(grid.t_frames)
    keys = [t for j in idx_row if j >= 0 for t in mem[j]]
    logits = [scale * sum(q[b, n, h, d] * k[b, t, h, d] for d in range(q.shape[-1])) for t in keys]
    m = max(logits)
    e = [math.exp(z - m) for z in logits]
    s = sum(e)
    out = [sum(e[a] / s * v[b, t, h, d] for a, t in enumerate(keys)) for d in range(q.shape[-1])]
    return out, m + math.log(s), [z / s for z in e]


def test_attend_brute_force_tokens():
    w, x = _inputs("tiny_ragged")
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, _, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    o, lse, probs = oracle.attend(x["q"], x["k"], x["v"], idx, g, scale, return_probs=True)
    mem = g.block_members(g.t_frames)
    for (b, h, i) in [(0, 0, 0), (0, 1, 3), (0, 1, g.nbq - 1)]:
        for pos, n in enumerate(mem[i][:5]):
            ref, ref_lse, ref_p = _brute_attend_token(x["q"], x["k"], x["v"], idx[b, h, i], g,
                                                      b, h, n, scale)
            np.testing.assert_allclose(o[b, n, h], ref, atol=1e-12)
            assert lse[b, n, h] == pytest.approx(ref_lse, rel=1e-12)
            np.testing.assert_allclose(probs[(b, h, i)][pos], ref_p, atol=1e-14)


def test_softmax_rows_sum_to_one_and_special_values():
    w, x = _inputs("tiny_ragged")
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, _, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    _, _, probs = oracle.attend(x["q"], x["k"], x["v"], idx, g, scale, return_probs=True)
    for p in probs.values():
        assert np.max(np.abs(p.sum(axis=1) - 1.0)) < 1e-12
        assert np.all(p >= 0)
    # V == c gives O == c
    vc = np.full_like(x["v"], 0.75)
    o, _ = oracle.attend(x["q"], x["k"], vc, idx, g, scale)
    np.testing.assert_allclose(o, 0.75, atol=1e-14)
    # Q == 0 gives the mean of the selected valid V rows
    o0, _ = oracle.attend(np.zeros_like(x["q"]), x["k"], x["v"], idx, g, scale)
    mem = g.block_members(g.t_frames)
    sel = [t for j in idx[0, 1, 2] if j >= 0 for t in mem[j]]
    np.testing.assert_allclose(o0[0, mem[2][0], 1], x["v"][0, sel, 1].mean(axis=0), atol=1e-13)


def test_continuation_cache_equals_full_grid():
    """Without the causal mask, a cached run equals a plain run on the whole key grid whose
    query rows are the last frames."""
    w, x = _inputs("small_cont")
    g = _grid(w)
    gf = Grid(w.t_frames + w.cached_t, w.grid_h, w.grid_w, w.blk)  # full grid, no cache
    g0 = Grid(w.t_frames, w.grid_h, w.grid_w, w.blk, w.cached_t, 0)
    scale = 1.0 / math.sqrt(w.head_dim)
    kf = np.concatenate([x["kc"], x["k"]], axis=1)
    vf = np.concatenate([x["vc"], x["v"]], axis=1)
    nc = w.n_cached_tokens
    qf = np.concatenate([np.zeros_like(x["kc"]), x["q"]], axis=1)
    idx, cnt, s = oracle.route(x["q"], x["k"], g0, w.top_r, k_cache=x["kc"])
    # same selections on the full grid: query block i of the cached run is block i + nbc
    idx_f = -np.ones((w.batch, w.heads, gf.nbq, w.top_r), dtype=np.int32)
    idx_f[:, :, g0.nbc:] = idx
    o, lse = oracle.attend(x["q"], x["k"], x["v"], idx, g0, scale, k_cache=x["kc"], v_cache=x["vc"])
    qb = [(b, h, i) for b in range(w.batch) for h in range(w.heads) for i in range(g0.nbc, gf.nbq)]
    of, lsef = oracle.attend(qf, kf, vf, idx_f, gf, scale, query_blocks=qb)
    np.testing.assert_allclose(o, of[:, nc:], atol=1e-12)
    np.testing.assert_allclose(lse, lsef[:, nc:], atol=1e-12)
    # and the routing scores on the full grid agree for the query rows
    qbar_full = oracle.block_means(qf, gf.block_members(gf.t_frames))
    kbar_full = oracle.block_means(kf, gf.block_members(gf.t_frames))
    s_full = np.einsum("bhid,bhjd->bhij", qbar_full, kbar_full)
    np.testing.assert_allclose(s, s_full[:, :, g0.nbc:], rtol=1e-12, atol=1e-14)
    assert g.nbc == g0.nbc


# ------------------------------------------------------------------ backward pins
@pytest.mark.parametrize("name", ["tiny", "tiny_ragged"])
def test_bwd_matches_torch_autograd_masked(name):
    w, x = _inputs(name)
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    for r in (w.top_r, g.nbk):
        idx, _, _ = oracle.route(x["q"], x["k"], g, r)
        dq, dk, dv = oracle.attend_bwd(x["q"], x["k"], x["v"], x["do"], idx, g, scale)
        mask = _token_mask(g, idx, w.batch, w.heads)
        o, (tq, tk, tv) = _sdpa(x["q"], x["k"], x["v"], scale, mask=mask, need_grad=True)
        tdo = torch.tensor(x["do"].transpose(0, 2, 1, 3).copy(), dtype=torch.float64)
        (o * tdo).sum().backward()
        for mine, t in ((dq, tq), (dk, tk), (dv, tv)):
            np.testing.assert_allclose(mine, t.grad.numpy().transpose(0, 2, 1, 3), atol=1e-11)


def test_bwd_finite_differences():
    w, x = _inputs("tiny_ragged")
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, _, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    dq, dk, dv = oracle.attend_bwd(x["q"], x["k"], x["v"], x["do"], idx, g, scale)
    rng = np.random.default_rng(17)
    eps = 1e-5

    def loss(q, k, v):
        o, _ = oracle.attend(q, k, v, idx, g, scale)
        return float(np.sum(o * x["do"]))
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        for _ in range(12):
            pos = tuple(int(rng.integers(0, s)) for s in x[name].shape)
            args = {"q": x["q"].copy(), "k": x["k"].copy(), "v": x["v"].copy()}
            args[name][pos] += eps
            lp = loss(args["q"], args["k"], args["v"])
            args[name][pos] -= 2 * eps
            lm = loss(args["q"], args["k"], args["v"])
            num = (lp - lm) / (2 * eps)
            assert grad[pos] == pytest.approx(num, rel=1e-6, abs=1e-8)


def test_bwd_continuation_grads_only_reach_current_keys():
    w, x = _inputs("small_cont")
    g = _grid(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, _, _ = oracle.route(x["q"], x["k"], g, w.top_r, k_cache=x["kc"])
    dq, dk, dv = oracle.attend_bwd(x["q"], x["k"], x["v"], x["do"], idx, g, scale,
                                   k_cache=x["kc"], v_cache=x["vc"])
    # full-grid autograd with the cache as part of the keys; compare current-key gradients
    nc = w.n_cached_tokens
    gf = Grid(w.t_frames + w.cached_t, w.grid_h, w.grid_w, w.blk)
    kf = np.concatenate([x["kc"], x["k"]], axis=1)
    vf = np.concatenate([x["vc"], x["v"]], axis=1)
    qf = np.concatenate([np.zeros_like(x["kc"]), x["q"]], axis=1)
    dof = np.concatenate([np.zeros_like(x["kc"]), x["do"]], axis=1)
    idx_f = -np.ones((w.batch, w.heads, gf.nbq, w.top_r), dtype=np.int32)
    idx_f[:, :, g.nbc:] = idx
    mask = _token_mask(gf, idx_f, w.batch, w.heads)
    mask[:, :, :nc, :nc] = True  # cached query rows are discarded; keep their softmax finite
    o, (tq, tk, tv) = _sdpa(qf, kf, vf, scale, mask=mask, need_grad=True)
    tdo = torch.tensor(dof.transpose(0, 2, 1, 3).copy(), dtype=torch.float64)
    (o * tdo).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy().transpose(0, 2, 1, 3)[:, nc:], atol=1e-11)
    np.testing.assert_allclose(dk, tk.grad.numpy().transpose(0, 2, 1, 3)[:, nc:], atol=1e-11)
    np.testing.assert_allclose(dv, tv.grad.numpy().transpose(0, 2, 1, 3)[:, nc:], atol=1e-11)


# ------------------------------------------------------------------ prologue backward
def _prologue_case(seed=5, frames=2, gh=3, gw=5, heads=2, d=12):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((1, frames * gh * gw, heads, d))
    gamma = 1.0 + 0.5 * rng.standard_normal(d)
    dz = rng.standard_normal(x.shape)
    return rng, x, gamma, dz


def test_prologue_bwd_finite_differences():
    """dx and dgamma against central differences of sum(dz * prologue(x; gamma))."""
    rng, x, gamma, dz = _prologue_case()
    kw = dict(eps=1e-6, theta=10.0, t_offset=3)
    dx, dgamma = oracle.prologue_bwd(dz, x, 2, 3, 5, gamma=gamma, **kw)

    def loss(xx, gg):
        return float(np.sum(dz * oracle.prologue(xx, 2, 3, 5, gamma=gg, **kw)))
    h = 1e-6
    for _ in range(16):
        pos = tuple(int(rng.integers(0, s)) for s in x.shape)
        xp, xm = x.copy(), x.copy()
        xp[pos] += h
        xm[pos] -= h
        assert dx[pos] == pytest.approx((loss(xp, gamma) - loss(xm, gamma)) / (2 * h), rel=1e-6, abs=1e-8)
    for dd in range(x.shape[-1]):
        gp, gm = gamma.copy(), gamma.copy()
        gp[dd] += h
        gm[dd] -= h
        assert dgamma[dd] == pytest.approx((loss(x, gp) - loss(x, gm)) / (2 * h), rel=1e-6, abs=1e-8)


def test_rope_transpose_undoes_the_rotation():
    """RoPE turns each pair by an angle, so its transpose is its inverse: rotating the
    transposed gradient forward gives it back, and pair norms are kept."""
    _, _, _, dz = _prologue_case(seed=8)
    t, h, w = oracle.grid_positions(2, 3, 5, t_offset=1)
    dy = oracle.rope3d_transpose(dz, t, h, w, 10000.0)
    np.testing.assert_allclose(oracle.rope3d(dy, t, h, w, 10000.0), dz, rtol=0, atol=1e-12)
    np.testing.assert_allclose(dy[..., 0::2] ** 2 + dy[..., 1::2] ** 2,
                               dz[..., 0::2] ** 2 + dz[..., 1::2] ** 2, rtol=1e-12, atol=1e-12)


def test_rmsnorm_bwd_is_orthogonal_to_the_input_without_eps():
    """With eps = 0 the normalised output does not change when x is scaled, so the gradient
    of any loss through it is orthogonal to x, row by row."""
    _, x, gamma, dz = _prologue_case(seed=9)
    dx, _ = oracle.rms_norm_bwd(dz, x, gamma, 0.0)
    np.testing.assert_allclose(np.sum(dx * x, axis=-1), 0.0, atol=1e-12)
    # and without a gain and without RoPE the prologue backward is the plain identity
    dx2, dg2 = oracle.prologue_bwd(dz, x, 2, 3, 5, gamma=None, theta=0.0)
    assert dg2 is None
    np.testing.assert_array_equal(dx2, dz)


# ------------------------------------------------------------------ routing variants
def _brute_variant(q, k, grid, r, pool, force_self, shared):
    """Scalar loops: per-head block pooling (mean / sum / channel max), scores, optional sum
    over heads, then the best-scoring set by exhaustive search over combinations (inputs are
    continuous random values, so the best set is unique), holding the own block when forced.
    Grids here have no cache, so query block i's own key block is block i."""
    B, N, H, D = q.shape
    mem = grid.block_members(grid.t_frames)

    def pooled(arr, b, h, toks):
        out = []
        for d in range(D):
            vals = [float(arr[b, t, h, d]) for t in toks]
            out.append(max(vals) if pool == "max" else sum(vals) / (len(vals) if pool == "mean" else 1))
        return out

    res = {}
    for b in range(B):
        per_head = []
        for h in range(H):
            qp = [pooled(q, b, h, t) for t in mem]
            kp = [pooled(k, b, h, t) for t in mem]
            per_head.append([[sum(qp[i][d] * kp[j][d] for d in range(D)) for j in range(grid.nbk)]
                             for i in range(grid.nbq)])
        if shared:
            per_head = [[[sum(per_head[h][i][j] for h in range(H)) for j in range(grid.nbk)]
                         for i in range(grid.nbq)]]
        for hh, sc in enumerate(per_head):
            for i in range(grid.nbq):
                allowed = [j for j in range(grid.nbk)
                           if not (grid.masked and grid.key_block_chunk(j) > grid.query_block_chunk(i))]
                must = [i] if force_self else []
                rest = [j for j in allowed if j not in must]
                m = min(r, len(allowed)) - len(must)
                best = max(itertools.combinations(rest, m), key=lambda c: sum(sc[i][j] for j in c))
                res[(b, hh, i)] = sorted(must + list(best))
    return res


@pytest.mark.parametrize("gridspec", [(4, 8, 8, 0), (3, 7, 6, 0), (8, 4, 4, 4)])
@pytest.mark.parametrize("pool,force_self,shared", [
    ("mean", True, False), ("mean", False, True), ("mean", True, True),
    ("sum", False, False), ("max", False, False), ("max", True, True)])
def test_route_variants_brute_force(gridspec, pool, force_self, shared):
    t, gh, gw, chunk = gridspec
    g = Grid(t, gh, gw, (2, 4, 4), chunk_t=chunk)
    rng = np.random.default_rng(17)
    q = rng.standard_normal((1, t * gh * gw, 2, 8))
    k = rng.standard_normal((1, t * gh * gw, 2, 8))
    r = 3
    idx, cnt, s = oracle.route(q, k, g, r, pool=pool, force_self=force_self, shared_heads=shared)
    ref = _brute_variant(q, k, g, r, pool, force_self, shared)
    for h in range(2):
        for i in range(g.nbq):
            sel = ref[(0, 0 if shared else h, i)]
            assert cnt[0, h, i] == len(sel)
            assert list(idx[0, h, i, :len(sel)]) == sel and all(idx[0, h, i, len(sel):] == -1)
            if force_self:
                assert i in sel
    if shared:
        assert s.shape[1] == 1 and np.array_equal(idx[:, 0], idx[:, 1])


def test_force_self_with_r1_keeps_only_the_own_block():
    w, x = _inputs("small_cont")
    g = _grid(w)
    idx, cnt, _ = oracle.route(x["q"], x["k"], g, 1, k_cache=x["kc"], force_self=True)
    assert np.all(cnt == 1)
    assert np.array_equal(idx[0, 0, :, 0], g.nbc + np.arange(g.nbq))


def test_force_self_changes_nothing_where_the_own_block_already_wins():
    w, x = _inputs("small")
    g = _grid(w)
    plain, _, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    forced, _, _ = oracle.route(x["q"], x["k"], g, w.top_r, force_self=True)
    has_own = np.array([[[i in plain[b, h, i] for i in range(g.nbq)] for h in range(w.heads)]
                        for b in range(w.batch)])
    assert has_own.any() and (~has_own).any()
    assert np.array_equal(plain[has_own], forced[has_own])
    assert not np.array_equal(plain[~has_own], forced[~has_own])


def test_shared_heads_with_identical_heads_is_the_per_head_route():
    w, x = _inputs("small_b2")
    g = _grid(w)
    q = np.repeat(x["q"][:, :, :1], w.heads, axis=2)
    k = np.repeat(x["k"][:, :, :1], w.heads, axis=2)
    per, _, s1 = oracle.route(q, k, g, w.top_r)
    sh, _, s = oracle.route(q, k, g, w.top_r, shared_heads=True)
    assert np.array_equal(per, sh)
    np.testing.assert_allclose(s[:, 0], w.heads * s1[:, 0], rtol=1e-12)


def test_pooling_modes_closed_forms():
    g = Grid(3, 7, 6, (2, 4, 4))  # ragged in t, h and w
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1, 3 * 7 * 6, 2, 8))
    mem = g.block_members(3)
    mean, tot, mx = (oracle.block_pool(x, mem, m) for m in ("mean", "sum", "max"))
    counts = np.array([len(m) for m in mem], dtype=np.float64)
    np.testing.assert_allclose(tot, mean * counts[None, None, :, None], rtol=1e-12)
    assert np.all(mx >= mean - 1e-15)
    # a block whose tokens all hold one vector pools to that vector in every mode
    x[0, mem[4]] = x[0, mem[4][0]]
    for m in ("mean", "max"):
        np.testing.assert_allclose(oracle.block_pool(x, mem, m)[0, :, 4], x[0, mem[4][0]], rtol=1e-15)
    # channel max commutes with adding a constant and with a token permutation
    perm = rng.permutation(x.shape[1])
    inv = np.argsort(perm)
    mem_p = [[int(inv[t]) for t in m] for m in mem]
    np.testing.assert_array_equal(oracle.block_pool(x[:, perm], mem_p, "max"), oracle.block_pool(x, mem, "max"))
    np.testing.assert_allclose(oracle.block_pool(x + 3.0, mem, "max"), oracle.block_pool(x, mem, "max") + 3.0)


def test_sum_pooling_ranks_like_mean_on_whole_blocks_and_penalises_partial_ones():
    w, x = _inputs("small")  # 10 x 20 grid: ragged blocks on h and w
    g = _grid(w)
    mem = g.block_members(w.t_frames)
    whole = [j for j, m in enumerate(mem) if len(m) == g.bs]
    part = [j for j, m in enumerate(mem) if len(m) < g.bs]
    assert whole and part
    _, _, sm = oracle.route(x["q"], x["k"], g, w.top_r)
    _, _, ss = oracle.route(x["q"], x["k"], g, w.top_r, pool="sum")
    counts = np.array([len(m) for m in mem], dtype=np.float64)
    np.testing.assert_allclose(ss, sm * counts[None, None, :, None] * counts[None, None, None, :],
                               rtol=1e-9, atol=1e-12)
    # among whole key blocks the order of scores is the same
    for i in range(g.nbq):
        a = np.argsort(-sm[0, 0, i, whole], kind="stable")
        b = np.argsort(-ss[0, 0, i, whole], kind="stable")
        assert np.array_equal(a, b)


# ------------------------------------------------------------------ two-segment block-causal mask
def test_two_segment_mask_brute_force():
    """Conditioning frames [0, cond_t) see only themselves; later frames see everything.  The
    allowed set is written here from that sentence alone (no segment function)."""
    g = Grid(8, 4, 8, (2, 4, 4), cond_t=4)  # 4 block-frames x 2 blocks; blocks 0-3 conditioning
    rng = np.random.default_rng(21)
    q = rng.standard_normal((1, 8 * 32, 1, 8))
    k = rng.standard_normal((1, 8 * 32, 1, 8))
    r = 3
    idx, cnt, s = oracle.route(q, k, g, r)
    mem = g.block_members(8)
    t0 = [min(t // 32 for t in m) for m in mem]  # first frame of each block (32 tokens per frame)
    qbar = [q[0, m, 0].mean(axis=0) for m in mem]
    kbar = [k[0, m, 0].mean(axis=0) for m in mem]
    for i in range(g.nbq):
        allowed = [j for j in range(g.nbk) if t0[i] >= 4 or t0[j] < 4]
        sc = {j: float(qbar[i] @ kbar[j]) for j in allowed}
        best = sorted(sorted(allowed, key=lambda j: (-sc[j], j))[:r])
        assert list(idx[0, 0, i, :cnt[0, 0, i]]) == best
        assert all(np.isneginf(s[0, 0, i, j]) for j in range(g.nbk) if j not in allowed)
    assert list(cnt[0, 0]) == [3, 3, 3, 3, 3, 3, 3, 3] and set(idx[0, 0, 0]) <= {0, 1, 2, 3}


def test_two_segment_conditioning_rows_ignore_the_generated_frames():
    """Changing the frames after cond_t changes nothing for the conditioning rows, which equal
    a plain run over the conditioning frames alone; with chunk = cond_t = half the frames the
    form equals two causal chunks."""
    w, x = _inputs("small")  # 8 frames, 10 x 20 grid, blocks 4x4x8
    g = Grid(8, 10, 20, (4, 4, 8), cond_t=4)
    scale = 1.0 / math.sqrt(w.head_dim)
    idx, cnt, _ = oracle.route(x["q"], x["k"], g, w.top_r)
    o, lse = oracle.attend(x["q"], x["k"], x["v"], idx, g, scale)
    ncond = 4 * 10 * 20
    q2, k2, v2 = (a.copy() for a in (x["q"], x["k"], x["v"]))
    rng = np.random.default_rng(4)
    for a in (q2, k2, v2):
        a[:, ncond:] = rng.standard_normal(a[:, ncond:].shape)
    idx2, _, _ = oracle.route(q2, k2, g, w.top_r)
    o2, _ = oracle.attend(q2, k2, v2, idx2, g, scale)
    per_t = g.nbh * g.nbw
    assert np.array_equal(idx[:, :, :per_t], idx2[:, :, :per_t])
    np.testing.assert_array_equal(o[:, :ncond], o2[:, :ncond])
    gc = Grid(4, 10, 20, (4, 4, 8))
    sl = (slice(None), slice(0, ncond))
    idc, _, _ = oracle.route(x["q"][sl], x["k"][sl], gc, w.top_r)
    assert np.array_equal(idc, idx[:, :, :per_t])
    oc, lsec = oracle.attend(x["q"][sl], x["k"][sl], x["v"][sl], idc, gc, scale)
    np.testing.assert_allclose(oc, o[:, :ncond], atol=1e-13)
    np.testing.assert_allclose(lsec, lse[:, :ncond], atol=1e-13)
    gchunk = Grid(8, 10, 20, (4, 4, 8), chunk_t=4)
    idk, _, _ = oracle.route(x["q"], x["k"], gchunk, w.top_r)
    assert np.array_equal(idk, idx)
    # the generated frames' rows are routed as without any mask
    idn, _, _ = oracle.route(x["q"], x["k"], Grid(8, 10, 20, (4, 4, 8)), w.top_r)
    assert np.array_equal(idn[:, :, per_t:], idx[:, :, per_t:])


def test_continuation_rounds_equal_one_causal_pass():
    """Three rounds of 4 frames, each with the earlier frames as its cache, against one pass
    over all 12 frames with 4-frame causal chunks: same selections (global key-block ids) and
    the same O / LSE on every round's rows."""
    rng = np.random.default_rng(8)
    T, gh, gw, blk, r = 12, 6, 12, (4, 4, 8), 3
    D = 16
    q, k, v = (rng.standard_normal((1, T * gh * gw, 2, D)) for _ in range(3))
    full = Grid(T, gh, gw, blk, chunk_t=4)
    scale = 1.0 / math.sqrt(D)
    idx_f, cnt_f, _ = oracle.route(q, k, full, r)
    o_f, lse_f = oracle.attend(q, k, v, idx_f, full, scale)
    per_round = 4 * gh * gw
    nb_round = full.nbq // 3
    for rd in range(3):
        g = Grid(4, gh, gw, blk, cached_t=4 * rd, chunk_t=4)
        cur = slice(rd * per_round, (rd + 1) * per_round)
        past = slice(0, rd * per_round)
        kc = k[:, past] if rd else None
        vc = v[:, past] if rd else None
        idx, cnt, _ = oracle.route(q[:, cur], k[:, cur], g, r, k_cache=kc)
        rows = slice(rd * nb_round, (rd + 1) * nb_round)
        assert np.array_equal(idx, idx_f[:, :, rows]) and np.array_equal(cnt, cnt_f[:, :, rows])
        o, lse = oracle.attend(q[:, cur], k[:, cur], v[:, cur], idx, g, scale, k_cache=kc, v_cache=vc)
        np.testing.assert_allclose(o, o_f[:, cur], atol=1e-12)
        np.testing.assert_allclose(lse, lse_f[:, cur], atol=1e-12)
