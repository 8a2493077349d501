"""GPU parity of the forward path (prologue -> route -> sparse attention) against the oracle.

Parity is staged so one stage's bf16 rounding never masquerades as the next stage's error:
the prologue is compared with the oracle's fp64 prologue (<= 1 bf16 ulp + 1e-5); the oracle's
route is fed the GPU's bf16 post-prologue q/k (selections must match exactly, except where
the oracle's scores put the swapped blocks within 1e-4 relative of the r-th score); the
oracle's attention is fed the GPU's q/k/v and the GPU's (checked) selections, and O must
match within max-abs 2e-2 and mean-abs 2e-3 over valid elements, LSE within 2e-3.
Small workloads are compared in full; the measured 480p / 720p / continuation workloads
are compared on sampled heads and query blocks in the same launch configuration the bench
uses.
"""
import math

import numpy as np
import pytest

import oracle
from synth import WORKLOADS, bf16_bits_to_f64, make_raster_inputs
from tests.helpers import bf16_dev_to_f64, bf16_ulp, blocked_to_raster, grid_of, to_dev

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 2e-3
PROLOGUE_ABS = 1e-5


@pytest.fixture(scope="module")
def torch_cuda():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch


def run_forward(w, x=None, top_r=None):
    import torch
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.pipeline import BsaPipeline
    x = x if x is not None else make_raster_inputs(w)
    g = bsa.Geometry.from_workload(w)
    pipe = BsaPipeline(g, top_r or w.top_r, rope_theta=w.theta if w.rope else 0.0,
                       qknorm=w.qknorm, eps=w.eps)
    if w.qknorm:
        pipe.set_gamma(to_dev(x["gamma_q"]), to_dev(x["gamma_k"]))
    if w.cached_t:
        pipe.load_cache(to_dev(x["kc"]), to_dev(x["vc"]))
    pipe.forward(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]))
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == 0
    return pipe, x


def head_raster(t, sm, h):
    """GPU blocked tensor -> fp64 raster [B, N, 1, D] of head h."""
    return blocked_to_raster(bf16_dev_to_f64(t[:, h:h + 1]), sm)


def check_prologue(w, pipe, x, heads):
    grid = grid_of(w)
    sm = grid.slot_map(w.t_frames)
    theta = w.theta if w.rope else 0.0
    for name, gam in (("q", x["gamma_q"]), ("k", x["gamma_k"]), ("v", None)):
        src = bf16_bits_to_f64(x[name])[:, :, heads]
        if name == "v":
            exp = src
        else:
            exp = oracle.prologue(src, w.t_frames, w.grid_h, w.grid_w,
                                  gamma=gam if w.qknorm else None, eps=w.eps, theta=theta,
                                  t_offset=w.cached_t)
        t = getattr(pipe, name)[:, heads]
        blk = bf16_dev_to_f64(t)
        got = blocked_to_raster(blk, sm)
        if name == "v":
            assert np.array_equal(got, exp)
        else:
            # one bf16 ulp of the exact value, plus the fp32 arithmetic's absolute error
            # (~1e-7 on O(1) normalised rows) where RoPE's two products nearly cancel
            err = np.abs(got - exp)
            tol = bf16_ulp(exp) + PROLOGUE_ABS
            assert np.all(err <= tol), f"{name}: max err/tol {np.max(err / tol)}"
        pad_b, pad_s = np.nonzero(sm < 0)
        assert np.all(blk[:, :, pad_b, pad_s, :] == 0.0)
    # block means written by the prologue = means of the GPU's own bf16 outputs
    for name, pool in (("q", pipe.q_pool), ("k", pipe.k_pool)):
        got = pool[:, heads].cpu().numpy().astype(np.float64)
        mine = oracle.block_means(blocked_to_raster(bf16_dev_to_f64(getattr(pipe, name)[:, heads]), sm),
                                  grid.block_members(w.t_frames))
        np.testing.assert_allclose(got, mine, rtol=2e-5, atol=2e-6)


def check_route(w, pipe, heads, rows=None):
    """Selections of the given heads (all query blocks, or `rows`) vs the oracle route fed
    with the GPU's post-prologue q/k.  Returns the number of near-tie exemptions."""
    grid = grid_of(w)
    sm = grid.slot_map(w.t_frames)
    idx_gpu = pipe.idx.cpu().numpy()
    cnt_gpu = pipe.cnt.cpu().numpy()
    exempt = 0
    for h in heads:
        q = head_raster(pipe.q, sm, h)
        k = head_raster(pipe.k, sm, h)
        kc = None
        if w.cached_t:
            kc = head_raster(pipe.kc, grid.slot_map(w.cached_t), h)
        ridx, rcnt, s = oracle.route(q, k, grid, pipe.r, k_cache=kc)
        for b in range(w.batch):
            for i in (rows if rows is not None else range(grid.nbq)):
                gsel, osel = idx_gpu[b, h, i], ridx[b, 0, i]
                assert cnt_gpu[b, h, i] == rcnt[b, 0, i], (b, h, i)
                assert np.all(gsel[cnt_gpu[b, h, i]:] == -1)
                if np.array_equal(gsel, osel):
                    continue
                assert np.all(np.diff(gsel[:cnt_gpu[b, h, i]]) > 0), "selection not ascending"
                assert oracle.near_tie_ok(gsel, osel, s[b, 0, i]), (b, h, i, gsel, osel)
                exempt += 1
    return exempt


def check_attention(w, pipe, heads, qblocks=None):
    grid = grid_of(w)
    sm = grid.slot_map(w.t_frames)
    idx_gpu = pipe.idx.cpu().numpy()
    errs = []
    for h in heads:
        q, k, v = (head_raster(getattr(pipe, n), sm, h) for n in ("q", "k", "v"))
        kc = vc = None
        if w.cached_t:
            smc = grid.slot_map(w.cached_t)
            kc, vc = head_raster(pipe.kc, smc, h), head_raster(pipe.vc, smc, h)
        qb = None
        if qblocks is not None:
            qb = [(b, 0, i) for b in range(w.batch) for i in qblocks]
        o_ref, lse_ref = oracle.attend(q, k, v, idx_gpu[:, h:h + 1], grid, pipe.g.scale,
                                       k_cache=kc, v_cache=vc, query_blocks=qb)
        o_blk = bf16_dev_to_f64(pipe.o[:, h:h + 1])
        o_gpu = blocked_to_raster(o_blk, sm)
        lse_blk = pipe.lse[:, h:h + 1].cpu().numpy().astype(np.float64)[..., None]
        lse_gpu = blocked_to_raster(lse_blk, sm)[..., 0]
        mem = grid.block_members(w.t_frames)
        toks = sorted(t for i in (qblocks if qblocks is not None else range(grid.nbq)) for t in mem[i])
        d = np.abs(o_gpu[:, toks] - o_ref[:, toks])
        errs.append(d)
        assert np.max(np.abs(lse_gpu[:, toks] - lse_ref[:, toks])) <= LSE_ABS
        pad_b, pad_s = np.nonzero(sm < 0)
        assert np.all(o_blk[:, :, pad_b, pad_s, :] == 0.0)
        assert np.all(np.isneginf(lse_blk[:, :, pad_b, pad_s, 0]))
    e = np.concatenate([x.reshape(-1) for x in errs])
    assert e.max() <= O_MAX_ABS, e.max()
    assert e.mean() <= O_MEAN_ABS, e.mean()
    return float(e.max()), float(e.mean())


SMALL = ["tiny", "tiny_ragged", "tiny_d128", "small", "small_b2", "small_cont", "small_cont_rope",
         "ragged_a", "ragged_b"]


@pytest.mark.parametrize("name", SMALL)
def test_forward_parity_small(torch_cuda, name):
    w = WORKLOADS[name]
    pipe, x = run_forward(w)
    heads = list(range(w.heads))
    check_prologue(w, pipe, x, heads)
    assert check_route(w, pipe, heads) == 0
    check_attention(w, pipe, heads)


@pytest.mark.parametrize("name", ["480p", "480p_cont", "720p"])
def test_forward_parity_full_size_sampled(torch_cuda, name):
    w = WORKLOADS[name]
    pipe, x = run_forward(w)
    grid = grid_of(w)
    rng = np.random.default_rng(123)
    heads = [0, int(rng.integers(1, w.heads))]
    rows = sorted(set(int(i) for i in rng.integers(0, grid.nbq, 48)) | {0, grid.nbq - 1})
    check_prologue(w, pipe, x, heads)
    exempt = check_route(w, pipe, heads, rows)
    assert exempt <= 1
    check_attention(w, pipe, heads, qblocks=rows[:16] + [grid.nbq - 1])


def _tiny_dup_inputs(w):
    """tiny-grid inputs where key blocks 1 and 5 are identical and query block 0 is aligned
    with them, so both tie for the top score of row 0 (layout-only prologue)."""
    x = make_raster_inputs(w)
    grid = grid_of(w)
    mem = grid.block_members(w.t_frames)
    k = x["k"].copy()
    k[:, mem[5]] = k[:, mem[1]]
    q = x["q"].copy()
    q[:, mem[0]] = k[:, mem[1]]
    x["k"], x["q"] = k, q
    return x


def test_route_exact_ties_lower_index(torch_cuda):
    w = WORKLOADS["tiny"]
    x = _tiny_dup_inputs(w)
    pipe, _ = run_forward(w, x=x, top_r=1)
    idx = pipe.idx.cpu().numpy()
    assert idx[0, 0, 0, 0] == 1 and idx[0, 1, 0, 0] == 1
    assert check_route(w, pipe, [0, 1]) == 0
    check_attention(w, pipe, [0, 1])


@pytest.mark.parametrize("r", [1, 8, 11])
def test_route_r_edge_cases(torch_cuda, r):
    """r = 1, r = NB (every block) and r > NB (cnt = NB, -1 padding)."""
    w = WORKLOADS["tiny_ragged"] if r == 1 else WORKLOADS["tiny"]
    pipe, _ = run_forward(w, top_r=r)
    nb = grid_of(w).nbk
    cnt = pipe.cnt.cpu().numpy()
    assert np.all(cnt == min(r, nb))
    if r >= nb:
        assert np.all(pipe.idx.cpu().numpy()[..., :nb] == np.arange(nb))
    assert check_route(w, pipe, list(range(w.heads))) == 0
    check_attention(w, pipe, list(range(w.heads)))


def test_partial_block_as_only_selection(torch_cuda):
    """A ragged key block (pads masked token-wise) as a query block's only selection."""
    from synth import bf16_bits_from_f32
    w = WORKLOADS["tiny_ragged"]
    grid = grid_of(w)
    mem = grid.block_members(w.t_frames)
    part = [j for j, m in enumerate(mem) if len(m) < grid.bs]
    assert part
    p = part[-1]
    x = make_raster_inputs(w)
    kbar = bf16_bits_to_f64(x["k"])[:, mem[p]].mean(axis=1)  # [B, H, D]
    q = bf16_bits_to_f64(x["q"])
    q[:, mem[0]] = 10.0 * kbar[:, None]
    x["q"] = bf16_bits_from_f32(q.astype(np.float32))
    pipe, _ = run_forward(w, x=x, top_r=1)
    assert check_route(w, pipe, list(range(w.heads))) == 0
    assert np.all(pipe.idx.cpu().numpy()[:, :, 0, 0] == p)
    check_attention(w, pipe, list(range(w.heads)))


def test_causal_fewer_allowed_than_r(torch_cuda):
    """Block-causal with a first chunk that allows fewer key blocks than r."""
    from synth import Workload
    w = Workload("causal_small", 1, 2, 128, 8, 8, 16, (4, 4, 8), 6, chunk_t=4, rope=True)
    pipe, _ = run_forward(w)
    grid = grid_of(w)
    cnt = pipe.cnt.cpu().numpy()
    per_chunk = grid.nbh * grid.nbw  # 4 blocks per t-block
    assert np.all(cnt[..., :per_chunk] == per_chunk)
    assert np.all(cnt[..., per_chunk:] == 6)
    idx = pipe.idx.cpu().numpy()
    for i in range(grid.nbq):
        sel = idx[0, :, i][idx[0, :, i] >= 0]
        assert np.all([grid.key_block_chunk(int(j)) <= grid.query_block_chunk(i) for j in sel])
    assert check_route(w, pipe, [0, 1]) == 0
    check_attention(w, pipe, [0, 1])


def test_bad_index_reports_status_without_fault(torch_cuda):
    import torch
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS["tiny"]
    pipe, _ = run_forward(w)
    pipe.idx[0, 0, 0, 0] = 999  # out of range: the kernel clamps, records, carries on
    pipe.attn_fwd()
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == 5
    assert bsa.bsa_device_status() == 0  # cleared


def test_bounded_wait_times_out_and_context_survives(torch_cuda):
    """A wait on a barrier that nothing signals gives up after its limit and reports
    BSA_ERR_TIMEOUT; the next launches on the same context still work and pass parity."""
    import time
    import block_sparse_attention_route_b200 as bsa
    t0 = time.perf_counter()
    bsa.bsa_selftest_bounded_wait(50000)  # 50 ms
    assert bsa.bsa_device_status() == 4
    assert time.perf_counter() - t0 < 5.0
    assert bsa.bsa_device_status() == 0
    w = WORKLOADS["tiny"]
    pipe, _ = run_forward(w)
    check_attention(w, pipe, [0, 1])


@pytest.mark.parametrize("cond_t,chunk_t", [(4, 0), (4, 4), (8, 0)])
def test_two_segment_mask(torch_cuda, cond_t, chunk_t):
    """Conditioning frames [0, cond_t) attend only among themselves; the frames after them
    attend to everything (or, with chunk_t, to their own and earlier chunks)."""
    from synth import Workload
    w = Workload("two_segment", 1, 2, 128, 12, 10, 20, (4, 4, 8), 5, chunk_t=chunk_t, rope=True,
                 cond_t=cond_t)
    pipe, _ = run_forward(w)
    grid = grid_of(w)
    idx = pipe.idx.cpu().numpy()
    per_t = grid.nbh * grid.nbw
    n_cond = (cond_t // 4) * per_t
    assert np.all(idx[:, :, :n_cond] < n_cond)  # conditioning rows never see later blocks
    assert np.any(idx[:, :, n_cond:] >= n_cond)
    assert check_route(w, pipe, [0, 1]) == 0
    check_attention(w, pipe, [0, 1])


@pytest.mark.parametrize("name", ["small", "small_b2", "small_cont_rope"])
def test_structured_inputs_parity(torch_cuda, name):
    """Inputs with a smooth field shared by q and k (video-like locality): the routing picks
    mostly neighbouring blocks; prologue, selections and attention still match the oracle."""
    from synth import add_smooth_field
    w = WORKLOADS[name]
    x = add_smooth_field(w, make_raster_inputs(w))
    pipe, _ = run_forward(w, x=x)
    heads = list(range(w.heads))
    check_prologue(w, pipe, x, heads)
    assert check_route(w, pipe, heads) == 0
    check_attention(w, pipe, heads)
