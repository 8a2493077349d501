"""GPU parity of the prologue backward (gradients through 3D RoPE and QK-RMSNorm to the raster
q, k, the gains, and the relayout of v) against the oracle's prologue_bwd.

Seeded synthetic gradients of the blocked outputs are made in raster order, relaid out on the
GPU by the forward prologue's v path (a pure relayout, checked by the prologue parity tests),
and the oracle gets the same bf16 values.  dx is compared per element within one bf16 ulp of
the reference plus 2e-5 (fp32 arithmetic, then rounding to bf16); dgamma (fp32 sums over every
token and head) within 1e-4 relative to the largest |dgamma| entry.  Pad slots of the blocked
gradients never reach the raster output.
"""
import numpy as np
import pytest

import oracle
from synth import WORKLOADS, bf16_bits_to_f64, make_raster_inputs, normal_bf16
from tests.helpers import bf16_dev_to_f64, bf16_ulp, to_dev

pytestmark = pytest.mark.gpu


def _relayout(g, frames, raster_dev):
    import torch
    import block_sparse_attention_route_b200 as bsa
    shp = bsa.blocked_shape(g, frames)
    out = torch.zeros(shp, dtype=torch.bfloat16, device="cuda")
    bsa.rope3d_qknorm_prologue(g, frames, 0, None, None, raster_dev, None, None, 0.0, 0.0,
                               None, None, out)
    return out


def run_case(name, with_gain=True, seed=40):
    import torch
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS[name]
    g = bsa.Geometry.from_workload(w)
    x = make_raster_inputs(w)
    shp = x["q"].shape
    dz = {t: normal_bf16(shp, seed + i) for i, t in enumerate(("q", "k", "v"))}
    gam = {"q": x["gamma_q"], "k": x["gamma_k"]} if (w.qknorm and with_gain) else {"q": None, "k": None}
    theta = w.theta if w.rope else 0.0
    dz_blk = {t: _relayout(g, w.t_frames, to_dev(dz[t])) for t in dz}
    dx = {t: torch.empty(shp, dtype=torch.bfloat16, device="cuda").view(torch.int16).fill_(0x7fc0)
              .view(torch.bfloat16) for t in dz}  # NaN-filled: every raster element must be written
    dgq = torch.full((w.head_dim,), float("nan"), device="cuda")
    dgk = torch.full((w.head_dim,), float("nan"), device="cuda")
    ws = torch.empty(max(bsa.bsa_workspace_size(g, 1, bsa.WS_PROLOGUE_BWD), 256), dtype=torch.uint8,
                     device="cuda")
    gq = None if gam["q"] is None else torch.from_numpy(gam["q"]).cuda()
    gk = None if gam["k"] is None else torch.from_numpy(gam["k"]).cuda()
    bsa.rope3d_qknorm_prologue_bwd(g, w.t_frames, w.cached_t, to_dev(x["q"]), to_dev(x["k"]), gq, gk,
                                   w.eps, theta, dz_blk["q"], dz_blk["k"], dz_blk["v"], dx["q"],
                                   dx["k"], dx["v"], dgq if gq is not None else None,
                                   dgk if gk is not None else None, ws)
    torch.cuda.synchronize()
    assert bsa.bsa_device_status() == 0
    for t in ("q", "k", "v"):
        got = bf16_dev_to_f64(dx[t])
        if t == "v":
            ref, dg = bf16_bits_to_f64(dz[t]), None
        else:
            ref, dg = oracle.prologue_bwd(bf16_bits_to_f64(dz[t]), bf16_bits_to_f64(x[t]), w.t_frames,
                                          w.grid_h, w.grid_w, gamma=gam[t], eps=w.eps, theta=theta,
                                          t_offset=w.cached_t)
        assert np.all(np.isfinite(got)), t
        err = np.abs(got - ref)
        bound = bf16_ulp(ref) + 2e-5
        assert np.all(err <= bound), (t, float(np.max(err - bound)))
        if dg is not None:
            dgg = (dgq if t == "q" else dgk).cpu().numpy().astype(np.float64)
            assert np.max(np.abs(dgg - dg)) <= 1e-4 * np.max(np.abs(dg)), (t, np.max(np.abs(dgg - dg)))


@pytest.mark.parametrize("name", ["small", "small_b2", "small_cont_rope", "tiny_ragged", "tiny_d128"])
def test_prologue_bwd_parity(name):
    run_case(name)


def test_prologue_bwd_without_gain_is_rope_transpose_and_relayout():
    run_case("small", with_gain=False)


def test_prologue_bwd_no_norm_no_rope_is_the_inverse_relayout():
    run_case("tiny")  # neither RMSNorm nor RoPE: dx is dz read back into raster order


def test_prologue_bwd_480p_sampled():
    """Full 480p size (32 heads x 37,440 tokens): all of dx and dgamma against the oracle."""
    run_case("480p")
