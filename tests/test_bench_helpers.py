"""Host-side arithmetic of bench.py (no GPU): the FLOP conventions, valid-token FLOPs from
the selections, per-block token counts, routing locality and the traffic scaling."""
import sys

import numpy as np
import pytest

import oracle
from synth import WORKLOADS


@pytest.fixture(scope="module")
def bench():
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        import bench as b
    finally:
        sys.argv = argv
    return b


def _geom(w):
    import block_sparse_attention_route_b200 as bsa
    return bsa.Geometry.from_workload(w)


@pytest.mark.parametrize("name", ["480p", "720p", "tiny_ragged", "small_b2"])
def test_block_token_counts_match_the_oracle_grid(bench, name):
    w = WORKLOADS[name]
    grid = oracle.Grid(w.t_frames, w.grid_h, w.grid_w, w.blk)
    got = bench.block_token_counts(_geom(w), w.t_frames)
    assert list(got) == [len(m) for m in grid.block_members(w.t_frames)]
    assert got.sum() == w.t_frames * w.grid_h * w.grid_w


def test_tile_flops_convention(bench):
    # 720p: 1,658,880 selected pairs of 128-token blocks at D = 128 -> 13.916 TFLOP
    assert bench.tile_flops(128, 128, 1658880) == pytest.approx(13.91569403904e12, rel=1e-12)


@pytest.mark.parametrize("name", ["small_cont", "tiny_ragged"])
def test_valid_token_flops_brute_force(bench, name):
    w = WORKLOADS[name]
    grid = oracle.Grid(w.t_frames, w.grid_h, w.grid_w, w.blk, w.cached_t, w.chunk_t)
    rng = np.random.default_rng(3)
    idx = np.sort(rng.choice(grid.nbk, size=(w.batch, w.heads, grid.nbq, w.top_r)), axis=-1).astype(np.int32)
    cnt = rng.integers(0, w.top_r + 1, size=(w.batch, w.heads, grid.nbq)).astype(np.int32)
    mq = grid.block_members(w.t_frames)
    nk = ([len(m) for m in grid.block_members(w.cached_t)] if w.cached_t else []) + [len(m) for m in mq]
    ref = sum(4 * w.head_dim * len(mq[i]) * nk[idx[b, h, i, e]]
              for b in range(w.batch) for h in range(w.heads) for i in range(grid.nbq)
              for e in range(cnt[b, h, i]))
    assert bench.valid_token_flops(_geom(w), idx, cnt) == ref


def test_selection_locality(bench):
    w = WORKLOADS["small"]  # 2 x 3 x 3 blocks
    g = _geom(w)
    nbq = 18
    # query block 0 at (0,0,0): blocks 1 (0,0,1) and 4 (0,1,1) are neighbours, 17 (1,2,2) is not
    idx = np.full((1, 1, nbq, 3), -1, dtype=np.int32)
    cnt = np.zeros((1, 1, nbq), dtype=np.int32)
    idx[0, 0, 0] = [1, 4, 17]
    cnt[0, 0, 0] = 3
    assert bench.selection_locality(g, idx, cnt) == pytest.approx(2 / 3)
    cnt[0, 0, 0] = 2  # only the first two count
    assert bench.selection_locality(g, idx, cnt) == 1.0


def test_traffic_scales_with_the_pairs_a_launch_reads(bench):
    assert bench.traffic_per_launch("fwd", "720p", 1000, 10) == bench.DRAM_BYTES_PER_PAIR["fwd"] * 1000
    assert bench.traffic_per_launch("bwd_dkdv", "720p", 1000, 10) == bench.DRAM_BYTES_PER_PAIR["bwd_dkdv"] * 10


def test_cpu_baseline_times_forward_and_backward(bench):
    """The oracle baseline reports the step's rate (forward + 2.5x forward tile FLOPs per query
    block over the oracle's forward + backward time per block) and both parts on their own;
    the step rate lies between the two parts' rates scaled by their FLOP shares."""
    cb = bench.cpu_oracle_sample(WORKLOADS["small"], budget_s=0.5, with_bwd=True)
    assert cb["kind"] == "oracle" and cb["unit"] == "TFLOP/s" and cb["cores"] >= 1
    assert cb["value"] > 0 and cb["fwd_tflops"] > 0 and cb["bwd_tflops"] > 0
    assert "backward of" in cb["sample"]
    # harmonic combination of the parts (route time makes the step rate a little lower)
    combined = 3.5 / (1.0 / cb["fwd_tflops"] + 2.5 / cb["bwd_tflops"])
    assert cb["value"] <= combined * 1.0001
    fwd_only = bench.cpu_oracle_sample(WORKLOADS["small"], budget_s=0.5, with_bwd=False)
    assert "bwd_tflops" not in fwd_only and "backward of" not in fwd_only["sample"]
