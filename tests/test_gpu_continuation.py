"""GPU parity of multi-round continuation against one pass of the oracle over the whole video.

Three rounds of 8 frames on a ragged 10 x 20 grid, block-causal with 4-frame chunks.  Round 0
has no cache; rounds 1 and 2 take as their cache what ``bsa_cache_append`` built from the
round before (blocked K, V and the key-block means), never the raster frames again.  Because
RoPE runs on absolute frame positions and the causal chunks are absolute, the rounds together
must give what one block-causal pass over all 24 frames gives: the oracle runs that single pass
(prologue in fp64; routing and attention fed the GPU's bf16 q / k / v, assembled over the
rounds) and each round is compared on its own query blocks.  The appended cache must equal the
earlier rounds' blocked K / V / means byte for byte.
"""
import numpy as np
import pytest

import oracle
from synth import Workload, bf16_bits_to_f64, make_raster_inputs
from tests.helpers import bf16_dev_to_f64, bf16_ulp, blocked_to_raster, grid_of, to_dev

pytestmark = pytest.mark.gpu

O_MAX_ABS, O_MEAN_ABS, LSE_ABS = 2e-2, 2e-3, 2e-3
ROUND_T, ROUNDS = 8, 3
FULL = Workload("cont3_full", 1, 2, 128, ROUND_T * ROUNDS, 10, 20, (4, 4, 8), 5, chunk_t=4,
                rope=True, qknorm=True, unit_gamma=False)


def round_workload(r):
    return Workload(f"cont3_r{r}", FULL.batch, FULL.heads, FULL.head_dim, ROUND_T, FULL.grid_h,
                    FULL.grid_w, FULL.blk, FULL.top_r, cached_t=ROUND_T * r, chunk_t=FULL.chunk_t,
                    rope=True, qknorm=True, unit_gamma=False)


def run_rounds(x):
    import torch
    import block_sparse_attention_route_b200 as bsa
    from block_sparse_attention_route_b200.pipeline import BsaPipeline
    hw = FULL.grid_h * FULL.grid_w
    pipes, caches, cache = [], [], None
    for r in range(ROUNDS):
        w = round_workload(r)
        pipe = BsaPipeline(bsa.Geometry.from_workload(w), w.top_r, rope_theta=w.theta,
                           qknorm=True, eps=w.eps)
        pipe.set_gamma(to_dev(x["gamma_q"]), to_dev(x["gamma_k"]))
        if cache is not None:
            pipe.set_cache(*cache)
        sl = slice(r * ROUND_T * hw, (r + 1) * ROUND_T * hw)
        pipe.forward(*(to_dev(np.ascontiguousarray(x[n][:, sl])) for n in ("q", "k", "v")))
        cache = pipe.next_round_cache()
        torch.cuda.synchronize()
        assert bsa.bsa_device_status() == 0
        pipes.append(pipe)
        caches.append(cache)
    return pipes, caches


def test_three_round_continuation_matches_one_causal_pass():
    x = make_raster_inputs(FULL)
    pipes, caches = run_rounds(x)
    full = grid_of(FULL)
    sm_r = grid_of(round_workload(0)).slot_map(ROUND_T)
    per_round = full.nbq // ROUNDS
    assert pipes[0].g.nbq == per_round

    # the appended caches are the rounds' own blocked tensors, byte for byte
    import torch
    bits = {torch.bfloat16: torch.int16, torch.float32: torch.int32}
    for r, (kc, vc, kp) in enumerate(caches):
        for got, name in ((kc, "k"), (vc, "v"), (kp, "k_pool")):
            exp = torch.cat([getattr(p, name) for p in pipes[:r + 1]], dim=2)
            assert torch.equal(got.view(bits[got.dtype]), exp.view(bits[exp.dtype])), (r, name)

    for h in range(FULL.heads):
        # prologue of each round = the single pass's prologue on that round's frames
        for name, gam in (("q", x["gamma_q"]), ("k", x["gamma_k"])):
            exp = oracle.prologue(bf16_bits_to_f64(x[name])[:, :, h:h + 1], FULL.t_frames,
                                  FULL.grid_h, FULL.grid_w, gamma=gam, eps=FULL.eps,
                                  theta=FULL.theta)
            got = np.concatenate([blocked_to_raster(bf16_dev_to_f64(getattr(p, name)[:, h:h + 1]),
                                                    sm_r) for p in pipes], axis=1)
            assert np.all(np.abs(got - exp) <= bf16_ulp(exp) + 1e-5), name

        q, k, v = (np.concatenate([blocked_to_raster(bf16_dev_to_f64(getattr(p, n)[:, h:h + 1]),
                                                     sm_r) for p in pipes], axis=1)
                   for n in ("q", "k", "v"))
        ridx, rcnt, s = oracle.route(q, k, full, FULL.top_r)
        idx_all = np.concatenate([p.idx[:, h:h + 1].cpu().numpy() for p in pipes], axis=2)
        cnt_all = np.concatenate([p.cnt[:, h:h + 1].cpu().numpy() for p in pipes], axis=2)
        assert np.array_equal(cnt_all, rcnt)
        for i in range(full.nbq):
            sel = idx_all[0, 0, i]
            if not np.array_equal(sel, ridx[0, 0, i]):
                assert oracle.near_tie_ok(sel, ridx[0, 0, i], s[0, 0, i]), (h, i, sel)
            # no round ever selects a key block of a later causal chunk
            assert all(full.key_block_chunk(int(j)) <= full.query_block_chunk(i)
                       for j in sel[sel >= 0])
        # rounds 1, 2 really route into their caches
        assert np.any(idx_all[0, 0, per_round:] < per_round)

        o_ref, lse_ref = oracle.attend(q, k, v, idx_all, full, pipes[0].g.scale)
        o_gpu = np.concatenate([blocked_to_raster(bf16_dev_to_f64(p.o[:, h:h + 1]), sm_r)
                                for p in pipes], axis=1)
        lse_gpu = np.concatenate([blocked_to_raster(
            p.lse[:, h:h + 1].cpu().numpy().astype(np.float64)[..., None], sm_r)[..., 0]
            for p in pipes], axis=1)
        d = np.abs(o_gpu - o_ref)
        assert d.max() <= O_MAX_ABS and d.mean() <= O_MEAN_ABS, (h, d.max(), d.mean())
        assert np.max(np.abs(lse_gpu - lse_ref)) <= LSE_ABS
