"""C-ABI library checks that need no GPU: it loads, exports every declared entry point,
and rejects bad arguments on the host before touching a device."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_route_b200 as bsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "bsa.h")).read()
    return re.findall(r"BSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert set(names) >= {"rope3d_qknorm_prologue", "bsa_route", "bsa_attn_fwd", "bsa_attn_bwd",
                          "bsa_workspace_size", "bsa_device_status", "bsa_error_string"}
    L = bsa.lib()
    for n in names:
        assert hasattr(L, n), n
    assert L.bsa_abi_version() == 2


def test_error_strings():
    for code in range(7):
        assert bsa.bsa_error_string(code)


def _g(**kw):
    base = dict(batch=1, heads=32, head_dim=128, t_frames=24, grid_h=45, grid_w=80)
    base.update(kw)
    return bsa.Geometry(**base)


def test_workspace_sizes_720p():
    g = _g()
    nbq = 720
    assert g.nbq == nbq
    route = bsa.bsa_workspace_size(g, 72, bsa.WS_ROUTE)
    assert route == 2 * 32 * nbq * 128 * 4
    assert bsa.bsa_workspace_size(g, 72, bsa.WS_FWD) == 0
    bwd = bsa.bsa_workspace_size(g, 72, bsa.WS_BWD)
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    rows = 32 * nbq * 128
    # -Delta and -log2 LSE per query row, reverse-index offsets and lists, the key-major
    # pass's hand-out order (one int per current key block), work counter
    assert bwd == (2 * up(rows * 4) + up(32 * (nbq + 1) * 4) + up(32 * nbq * 72 * 4)
                   + up(32 * nbq * 4) + 256)


@pytest.mark.parametrize("bad", [dict(head_dim=96), dict(blk=(4, 4, 4)), dict(cached_t=3),
                                 dict(causal_chunk_t=6), dict(cond_t=6), dict(cond_t=-4), dict(batch=0), dict(grid_w=0),
                                 dict(softmax_scale=-1.0)])
def test_bad_geometry_rejected_on_host(bad):
    g = _g(**bad)
    assert bsa.bsa_workspace_size(g, 8, bsa.WS_ROUTE) == 0
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_route(g, 8, 16, 16, None, None, None, 16, 16, None, stream=0)
    assert ei.value.code in (1, 2)


def test_bad_arguments_rejected_on_host():
    g = _g()
    with pytest.raises(bsa.BsaError) as ei:  # top_r < 1
        bsa.bsa_attn_fwd(g, 0, 16, 16, 16, None, None, 16, 16, 16, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # missing output
        bsa.bsa_attn_fwd(g, 8, 16, 16, 16, None, None, 16, 16, None, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # misaligned pointer
        bsa.bsa_attn_fwd(g, 8, 17, 16, 16, None, None, 16, 16, 16, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # cache geometry without cache tensors
        bsa.bsa_attn_fwd(_g(cached_t=12, t_frames=12), 8, 16, 16, 16, None, None, 16, 16, 16, 16,
                         stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # route without workspace
        bsa.bsa_route(g, 8, 16, 16, None, None, None, 16, 16, None, stream=0)
    assert ei.value.code == 6
    with pytest.raises(bsa.BsaError) as ei:  # prologue: output without input
        bsa.rope3d_qknorm_prologue(g, 24, 0, None, None, None, None, None, 1e-6, 1e4, 16, None,
                                   None, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # bwd workspace too small
        bsa.bsa_attn_bwd(g, 8, *([16] * 3), None, None, 16, 16, 16, 16, 16, 16, 16, 16, 16,
                         stream=0)
    assert ei.value.code == 6


def test_kernel_timing_bookkeeping_without_launches():
    # host-side only: nothing recorded, so nothing to wait for and all counts are zero
    bsa.bsa_kernel_timing(True)
    assert bsa.bsa_kernel_times() == {k: (0, 0.0) for k in bsa.TIMED_KERNELS}
    bsa.bsa_kernel_timing(False)
    assert bsa.bsa_kernel_times() == {k: (0, 0.0) for k in bsa.TIMED_KERNELS}
    assert bsa.bsa_kernel_time_stats() == {k: (0, 0.0, 0.0, 0.0) for k in bsa.TIMED_KERNELS}


def test_prologue_bwd_host_validation():
    g = _g()
    assert bsa.bsa_workspace_size(g, 1, bsa.WS_PROLOGUE_BWD) == 2 * (-(-(720 * 4 * 128 * 4) // 256) * 256)
    with pytest.raises(bsa.BsaError) as ei:  # nothing to process
        bsa.rope3d_qknorm_prologue_bwd(g, 24, 0, None, None, None, None, 1e-6, 1e4,
                                       None, None, None, None, None, None, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # a gradient without its output
        bsa.rope3d_qknorm_prologue_bwd(g, 24, 0, None, None, None, None, 1e-6, 1e4,
                                       16, None, None, None, None, None, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # a gain needs the raster input and a dgamma output
        bsa.rope3d_qknorm_prologue_bwd(g, 24, 0, None, None, 16, None, 1e-6, 1e4,
                                       16, None, None, 16, None, None, stream=0)
    assert ei.value.code == 1


def test_cache_append_host_validation():
    g = _g(cached_t=8)
    with pytest.raises(bsa.BsaError) as ei:  # a ragged last block-frame cannot extend a cache
        bsa.bsa_cache_append(_g(t_frames=23), 16, 16, 16, 16, 16, 16, 16, 16, 16, stream=0)
    assert ei.value.code == 2
    with pytest.raises(bsa.BsaError) as ei:  # cached blocks to copy but no cache given
        bsa.bsa_cache_append(g, None, None, None, 16, 16, 16, 16, 16, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # new block means without the current ones
        bsa.bsa_cache_append(g, 16, 16, 16, 16, 16, None, 16, 16, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # misaligned output
        bsa.bsa_cache_append(g, 16, 16, 16, 16, 16, 16, 24, 16, 16, stream=0)
    assert ei.value.code == 1


def test_route_variant_host_validation():
    g = _g()
    args = (16, 16, None, None, None, 16, 16, 16)
    with pytest.raises(bsa.BsaError) as ei:  # unknown flag bit
        bsa.bsa_route_ex(g, 4, 16, *args, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # two pooling modes
        bsa.bsa_route_ex(g, 4, bsa.ROUTE_POOL_SUM | bsa.ROUTE_POOL_MAX, *args, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # a pooling variant cannot take the prologue's means
        bsa.bsa_route_ex(g, 4, bsa.ROUTE_POOL_MAX, 16, 16, 16, 16, None, 16, 16, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # unknown pooling mode
        bsa.bsa_block_pool(g, 24, 3, 16, 16, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:
        bsa.bsa_block_pool(g, 0, bsa.POOL_MAX, 16, 16, stream=0)
    assert ei.value.code == 1


def test_sharded_relayout_host_validation():
    g = _g(heads=4)  # a rank's slice: 4 of 32 heads
    ok = bsa.Shards(8, 3, 32, 28)
    cases = [  # (shards, q shard list) -> expected code
        (bsa.Shards(9, 3, 32, 0), [16] * 9),    # more shards than supported
        (bsa.Shards(8, 2, 32, 0), [16] * 8),    # 8 x 2 frames != 24
        (bsa.Shards(8, 3, 32, 29), [16] * 8),   # heads 29..32 outside 0..31
        (bsa.Shards(8, 3, 2, 0), [16] * 8),     # fewer raster heads than the call's
        (ok, [16] * 7 + [None]),                # a missing shard
        (ok, [16] * 7 + [24]),                  # a misaligned shard
    ]
    for sh, qs in cases:
        with pytest.raises(bsa.BsaError) as ei:
            bsa.rope3d_qknorm_prologue_sharded(g, 24, 0, sh, qs, None, None, None, None, 1e-6,
                                               1e4, 16, None, None, stream=0)
        assert ei.value.code == 1, (sh, qs)
    with pytest.raises(bsa.BsaError) as ei:  # the inverse relayout needs its shard table
        bsa.bsa_blocked_to_raster_sharded(g, 24, ok, 16, None, stream=0)
    assert ei.value.code == 1
    with pytest.raises(bsa.BsaError) as ei:  # a gain needs the raster q shards
        bsa.rope3d_qknorm_prologue_bwd_sharded(g, 24, 0, ok, None, None, 16, None, 1e-6, 1e4,
                                               16, None, None, [16] * 8, None, None, 16, None,
                                               stream=0)
    assert ei.value.code == 1
