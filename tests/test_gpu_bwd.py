"""GPU parity of the sparse attention backward against the oracle's closed-form gradients.

The oracle is fed the GPU's bf16 post-prologue q/k/v, the GPU's routing and the bf16 dO the
GPU receives; dQ, dK, dV must match within max-abs 2e-2 and mean-abs 2e-3 over valid rows,
with pad rows exactly zero.  Small ragged / cached workloads are compared in full; the 480p
backward workload is compared on sampled heads (every query and key block of those heads).
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOADS, bf16_bits_to_f64, make_raster_inputs
from tests.helpers import bf16_dev_to_f64, blocked_to_raster, grid_of, to_dev

pytestmark = pytest.mark.gpu

MAX_ABS, MEAN_ABS = 2e-2, 2e-3


def run_fwd_bwd(w, top_r=None):
    import torch
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.pipeline import BsaPipeline
    x = make_raster_inputs(w, with_grad=True)
    g = bsa.Geometry.from_workload(w)
    pipe = BsaPipeline(g, top_r or w.top_r, rope_theta=w.theta if w.rope else 0.0,
                       qknorm=w.qknorm, eps=w.eps, with_bwd=True)
    if w.qknorm:
        pipe.set_gamma(to_dev(x["gamma_q"]), to_dev(x["gamma_k"]))
    if w.cached_t:
        pipe.load_cache(to_dev(x["kc"]), to_dev(x["vc"]))
    pipe.forward(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]))
    pipe.load_grad(to_dev(x["do"]))
    pipe.backward()
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == 0
    return pipe, x


def check_bwd(w, pipe, x, heads):
    grid = grid_of(w)
    sm = grid.slot_map(w.t_frames)
    idx = pipe.idx.cpu().numpy()
    errs = []
    for h in heads:
        q, k, v = (blocked_to_raster(bf16_dev_to_f64(getattr(pipe, n)[:, h:h + 1]), sm)
                   for n in ("q", "k", "v"))
        kc = vc = None
        if w.cached_t:
            smc = grid.slot_map(w.cached_t)
            kc = blocked_to_raster(bf16_dev_to_f64(pipe.kc[:, h:h + 1]), smc)
            vc = blocked_to_raster(bf16_dev_to_f64(pipe.vc[:, h:h + 1]), smc)
        do = bf16_bits_to_f64(x["do"][:, :, h:h + 1])
        dq, dk, dv = oracle.attend_bwd(q, k, v, do, idx[:, h:h + 1], grid, pipe.g.scale,
                                       k_cache=kc, v_cache=vc)
        pad_b, pad_s = np.nonzero(sm < 0)
        for name, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
            blk = bf16_dev_to_f64(getattr(pipe, name)[:, h:h + 1])
            assert np.all(blk[:, :, pad_b, pad_s, :] == 0.0), f"{name}: pad rows not zero"
            d = np.abs(blocked_to_raster(blk, sm) - ref)
            errs.append((name, d))
            assert d.max() <= MAX_ABS, (name, h, d.max())
    for name in ("dq", "dk", "dv"):
        e = np.concatenate([d.reshape(-1) for n, d in errs if n == name])
        assert e.mean() <= MEAN_ABS, (name, e.mean())
    return {n: float(np.max(d)) for n, d in errs}


def check_bwd_sampled(w, pipe, x, plan, seed):
    """Sampled backward parity.  ``plan`` lists (head, extra random key blocks); per head: dQ
    of 6 full and 2 partial query blocks, dK / dV of the key block with the longest reverse
    list, the least-selected one (exactly zero if no query block chose it), the most-selected
    partial block and the random extras.  The oracle runs only the query blocks that selected
    those key blocks (their dK / dV are then complete) and the dQ sample.  Returns the longest
    reverse list seen."""
    grid = grid_of(w)
    sm = grid.slot_map(w.t_frames)
    idx = pipe.idx.cpu().numpy()
    nbq = grid.nbq
    n_valid = (sm >= 0).sum(axis=1)
    partial = np.nonzero(n_valid < grid.bs)[0]
    full = np.setdiff1d(np.arange(nbq), partial)
    rng = np.random.default_rng(seed)
    errs = {"dq": [], "dk": [], "dv": []}
    longest = 0
    for h, n_rand in plan:
        sel = idx[0, h]
        uses = np.bincount(sel[sel >= 0], minlength=nbq)
        kb = [int(np.argmax(uses)), int(np.argmin(uses))]
        if partial.size:
            kb.append(int(partial[np.argmax(uses[partial])]))
        kb += [int(j) for j in rng.choice(np.setdiff1d(np.arange(nbq), kb), n_rand, replace=False)]
        qs = [int(i) for i in rng.choice(full, min(6, full.size), replace=False)]
        if partial.size:
            qs += [int(i) for i in rng.choice(partial, min(2, partial.size), replace=False)]
        longest = max(longest, int(uses.max()))
        need = set(qs)
        for j in kb:
            need |= set(np.nonzero((sel == j).any(axis=1))[0].tolist())
        q, k, v = (blocked_to_raster(bf16_dev_to_f64(getattr(pipe, n)[:, h:h + 1]), sm)
                   for n in ("q", "k", "v"))
        do = bf16_bits_to_f64(x["do"][:, :, h:h + 1])
        dq, dk, dv = oracle.attend_bwd(q, k, v, do, idx[:, h:h + 1], grid, pipe.g.scale,
                                       query_blocks=[(0, 0, i) for i in sorted(need)])
        got = {n: bf16_dev_to_f64(getattr(pipe, n)[:, h:h + 1]) for n in ("dq", "dk", "dv")}
        for name, ref, blocks in (("dq", dq, qs), ("dk", dk, kb), ("dv", dv, kb)):
            for b in blocks:
                tile = got[name][0, 0, b]
                pad = sm[b] < 0
                assert np.all(tile[pad] == 0.0), f"{name}: pad rows of block {b} not zero"
                if name != "dq" and uses[b] == 0:
                    assert np.all(tile == 0.0), f"{name}: unselected key block {b} not zero"
                d = np.abs(tile[~pad] - ref[0, sm[b][~pad], 0])
                assert d.max() <= MAX_ABS, (name, h, b, d.max())
                errs[name].append(d.reshape(-1))
    for name, e in errs.items():
        e = np.concatenate(e)
        assert e.mean() <= MEAN_ABS, (name, e.mean())
    return longest


def test_backward_720p_sampled_blocks():
    """The bench's 720p workload (24x45x80 tokens, 720 blocks of 4x4x8, r = 72, 32 heads x 128)
    forward and backward in the bench's launch configuration, checked on heads 0 and 21 (8 key
    blocks and 16 query blocks in all, see check_bwd_sampled); the dK/dV pass's long reverse
    lists (well over 150 query blocks) are among them."""
    w = WORKLOADS["720p"]
    pipe, x = run_fwd_bwd(w)
    assert check_bwd_sampled(w, pipe, x, ((0, 2), (21, 0)), seed=720) > 150


@pytest.mark.parametrize("name", ["small", "small_b2", "small_cont", "small_cont_rope", "ragged_a",
                                  "ragged_b"])
def test_backward_parity_small(name):
    w = WORKLOADS[name]
    pipe, x = run_fwd_bwd(w)
    check_bwd(w, pipe, x, list(range(w.heads)))


def test_backward_all_blocks_selected():
    """r >= number of key blocks: every block selected (dense attention per head)."""
    w = WORKLOADS["small"]
    nbq, _ = w.n_blocks()
    pipe, x = run_fwd_bwd(w, top_r=nbq + 3)
    assert np.all(pipe.cnt.cpu().numpy() == nbq)
    check_bwd(w, pipe, x, [0, 1])


def test_backward_top1_leaves_key_blocks_unselected():
    """r = 1: most key blocks are selected by no query block; their dK / dV rows must be exactly
    zero, and the work distribution of the dK/dV pass must skip them without stalling."""
    w = WORKLOADS["small"]
    pipe, x = run_fwd_bwd(w, top_r=1)
    idx = pipe.idx.cpu().numpy()
    assert np.unique(idx[idx >= 0]).size < pipe.g.nbq  # some blocks really are unselected
    check_bwd(w, pipe, x, list(range(w.heads)))


def test_backward_480p_sampled_heads():
    w = WORKLOADS["480p_bwd"]
    pipe, x = run_fwd_bwd(w)
    check_bwd(w, pipe, x, [0, 17])


def test_backward_unsupported_block_size_is_reported():
    import torch
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS["tiny"]
    g = bsa.Geometry.from_workload(w)
    t = torch.zeros(1024, device="cuda")
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_attn_bwd(g, 2, t, t, t, None, None, t, t, t, t, t, t, t, t,
                         torch.zeros(bsa.bsa_workspace_size(g, 2, bsa.WS_BWD), dtype=torch.uint8,
                                     device="cuda"))
    assert ei.value.code == 2


def test_kernel_timing_counts_each_attention_launch():
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS["small"]
    bsa.bsa_kernel_timing(True)
    try:
        run_fwd_bwd(w)
        t = bsa.bsa_kernel_times()
    finally:
        bsa.bsa_kernel_timing(False)
    assert {k: n for k, (n, _) in t.items()} == {"fwd": 1, "bwd_dkdv": 1, "bwd_dq": 1}
    assert all(ms > 0 for _, ms in t.values())


def test_kernel_time_stats_min_median():
    """Three forward launches: min <= median <= mean, all three counted."""
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS["small"]
    pipe, _ = run_fwd_bwd(w)
    bsa.bsa_kernel_timing(True)
    try:
        for _ in range(3):
            pipe.attn_fwd()
        st = bsa.bsa_kernel_time_stats()
    finally:
        bsa.bsa_kernel_timing(False)
    n, tot, mn, med = st["fwd"]
    assert n == 3 and st["bwd_dkdv"][0] == 0
    assert 0 < mn <= med <= tot / n * 1.5 and mn <= tot / n


def test_backward_two_segment_mask():
    from synth import Workload
    w = Workload("two_segment", 1, 2, 128, 12, 10, 20, (4, 4, 8), 5, rope=True, cond_t=4)
    pipe, x = run_fwd_bwd(w)
    check_bwd(w, pipe, x, [0, 1])
