"""bsa_route_noalloc: routing for callers that cannot allocate device memory (a serving engine
that reserved the whole device, a framework allocator that owns every byte, a latency path
where cudaMalloc could synchronise).  Its block means live in a fixed array inside the
library, so its results must equal bsa_route with a caller workspace, on consecutive calls
(the array keeps the previous call's contents).  Collected last on purpose; it also passes
alone in a fresh process, where its first call performs the per-device address lookup."""
import numpy as np
import pytest

from synth import WORKLOADS, make_raster_inputs
from tests.helpers import to_dev

pytestmark = pytest.mark.gpu


def _blocked_inputs(w):
    import torch
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.pipeline import BsaPipeline
    x = make_raster_inputs(w)
    g = bsa.Geometry.from_workload(w)
    pipe = BsaPipeline(g, w.top_r, rope_theta=w.theta if w.rope else 0.0, qknorm=w.qknorm,
                       eps=w.eps)
    if w.qknorm:
        pipe.set_gamma(to_dev(x["gamma_q"]), to_dev(x["gamma_k"]))
    if w.cached_t:
        pipe.load_cache(to_dev(x["kc"]), to_dev(x["vc"]))
    pipe.prologue(to_dev(x["q"]), to_dev(x["k"]), to_dev(x["v"]))
    torch.cuda.synchronize()
    return g, pipe


@pytest.mark.parametrize("name", ["small", "small_cont", "480p"])
def test_route_noalloc_matches_workspace_route_twice(name):
    import torch
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS[name]
    g, pipe = _blocked_inputs(w)
    # reference: the workspace entry point, means computed from the blocked tensors
    bsa.bsa_route(g, w.top_r, pipe.q, pipe.k, None, None, pipe.kc_pool, pipe.idx, pipe.cnt,
                  pipe.ws_route)
    torch.cuda.synchronize()
    ref_idx, ref_cnt = pipe.idx.cpu().numpy(), pipe.cnt.cpu().numpy()
    for _ in range(2):
        idx = torch.full_like(pipe.idx, -7)
        cnt = torch.full_like(pipe.cnt, -7)
        bsa.bsa_route_noalloc(g, w.top_r, pipe.q, pipe.k, pipe.kc_pool, idx, cnt)
        torch.cuda.synchronize()
        assert bsa.bsa_device_status() == 0
        # routing decisions are bit-exact: same kernels, same fp32 arithmetic
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
        np.testing.assert_array_equal(cnt.cpu().numpy(), ref_cnt)


def test_route_noalloc_rejects_too_large_geometry():
    import torch
    import block_sparse_attention_route_b200 as bsa
    w = WORKLOADS["720p"]  # 2 * 32 * 720 * 128 * 4 bytes of means > 16 MiB
    g = bsa.Geometry.from_workload(w)
    t = torch.zeros(1024, device="cuda")
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_route_noalloc(g, w.top_r, t, t, None, t, t)
    assert ei.value.code == 2
    assert "16777216" in str(ei.value)
