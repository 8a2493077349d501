"""Seeded synthetic workloads for block sparse attention over 3D latent video tokens.

This module holds no arithmetic of the method: it only names the workload shapes, draws
seeded standard-normal numbers and converts them to and from bf16 bit patterns.  Both the
fp64 oracle (through the tests) and the CUDA library (through the tests and the bench)
receive the *same bytes* from here.

Generator: NumPy ``Generator(PCG64(seed))``, float32 N(0, 1), rounded to bf16 with
round-to-nearest-even on the host.  Seeds: Q = 0, K = 1, V = 2, dO = 3, cached K = 6,
cached V = 7, RMSNorm gains = 8 (only where a workload asks for non-unit gains).
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

SEED_Q, SEED_K, SEED_V, SEED_DO, SEED_KC, SEED_VC, SEED_GAMMA = 0, 1, 2, 3, 6, 7, 8


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape of one synthetic BSA problem.

    ``t_frames`` latent frames of current tokens (queries and current keys) on a
    ``grid_h`` x ``grid_w`` grid; ``cached_t`` leading frames whose keys/values come from a
    cache; ``blk`` the 3D block (t, h, w); ``top_r`` key blocks kept per query block;
    ``chunk_t`` the block-causal chunk in frames (0 = no chunks); ``cond_t`` the leading
    conditioning frames of the two-segment block-causal form (0 = none).
    """
    name: str
    batch: int
    heads: int
    head_dim: int
    t_frames: int
    grid_h: int
    grid_w: int
    blk: tuple
    top_r: int
    cached_t: int = 0
    chunk_t: int = 0
    rope: bool = True
    qknorm: bool = True
    theta: float = 10000.0
    eps: float = 1e-6
    unit_gamma: bool = True
    cond_t: int = 0

    @property
    def n_tokens(self) -> int:
        return self.t_frames * self.grid_h * self.grid_w

    @property
    def n_cached_tokens(self) -> int:
        return self.cached_t * self.grid_h * self.grid_w

    def padded(self):
        bt, bh, bw = self.blk
        up = lambda x, b: -(-x // b) * b  # noqa: E731
        return up(self.t_frames, bt), up(self.grid_h, bh), up(self.grid_w, bw)

    def n_blocks(self):
        """(query blocks, cached key blocks) of the padded grid."""
        bt, bh, bw = self.blk
        tp, hp, wp = self.padded()
        per_t = (hp // bh) * (wp // bw)
        return (tp // bt) * per_t, (self.cached_t // bt) * per_t

    def block_size(self) -> int:
        return self.blk[0] * self.blk[1] * self.blk[2]


# The five workloads the method is measured on (tiny, 480p coarse, 720p refine, 480p
# continuation, 480p backward) plus small parity workloads that span several tiles and
# have ragged (padded) blocks, sized so the fp64 oracle finishes in seconds.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 64, 4, 8, 8, (2, 4, 4), 2, rope=False, qknorm=False),
    "480p": Workload("480p", 1, 32, 128, 24, 30, 52, (4, 4, 8), 34),
    "720p": Workload("720p", 1, 32, 128, 24, 45, 80, (4, 4, 8), 72),
    "480p_cont": Workload("480p_cont", 1, 32, 128, 12, 30, 52, (4, 4, 8), 34, cached_t=12,
                          chunk_t=4, rope=False, qknorm=False),
    "480p_bwd": Workload("480p_bwd", 1, 32, 128, 24, 30, 52, (4, 4, 8), 34),
    # small parity cases (not measured): ragged h and w, several tiles per head
    "small": Workload("small", 1, 2, 128, 8, 10, 20, (4, 4, 8), 4),
    "small_b2": Workload("small_b2", 2, 3, 128, 6, 9, 13, (4, 4, 8), 3, unit_gamma=False),
    "small_cont": Workload("small_cont", 1, 2, 128, 8, 10, 20, (4, 4, 8), 5, cached_t=8,
                           chunk_t=4, rope=False, qknorm=False),
    "small_cont_rope": Workload("small_cont_rope", 1, 2, 128, 8, 6, 12, (4, 4, 8), 3,
                                cached_t=4, chunk_t=8),
    "tiny_d128": Workload("tiny_d128", 1, 2, 128, 4, 8, 8, (2, 4, 4), 3),
    "tiny_ragged": Workload("tiny_ragged", 1, 2, 64, 3, 7, 6, (2, 4, 4), 2),
    # every class of valid count a partial 128-token block can have: 5x9x11 gives blocks of
    # 128, 48, 32, 12, 8 and 3 tokens; 7x11x13 gives 128, 96, 80, 72, 60 and 45
    "ragged_a": Workload("ragged_a", 1, 2, 128, 5, 9, 11, (4, 4, 8), 4),
    "ragged_b": Workload("ragged_b", 1, 2, 128, 7, 11, 13, (4, 4, 8), 5),
}


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); return the uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(bits).astype(np.float64)


def normal_bf16(shape, seed: int) -> np.ndarray:
    """Seeded N(0,1) float32 draws rounded to bf16; returns uint16 bit patterns."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return bf16_bits_from_f32(rng.standard_normal(size=shape, dtype=np.float32))


def make_raster_inputs(w: Workload, with_grad: bool = False,
                       seed_offset: int = 0) -> Dict[str, Optional[np.ndarray]]:
    """Raster inputs [B, N, H, D] (bf16 bits) in (t, h, w) row-major token order.

    Returns q, k, v (current frames), kc, vc (cached frames, or None), do (upstream
    gradient over the current query tokens, or None) and gamma_q, gamma_k (float32 [D]
    RMSNorm gains, or None when the workload has no QK-norm).
    """
    shp = (w.batch, w.n_tokens, w.heads, w.head_dim)
    out: Dict[str, Optional[np.ndarray]] = {
        "q": normal_bf16(shp, SEED_Q + seed_offset),
        "k": normal_bf16(shp, SEED_K + seed_offset),
        "v": normal_bf16(shp, SEED_V + seed_offset),
        "kc": None, "vc": None, "do": None, "gamma_q": None, "gamma_k": None,
    }
    if w.cached_t:
        cshp = (w.batch, w.n_cached_tokens, w.heads, w.head_dim)
        out["kc"] = normal_bf16(cshp, SEED_KC + seed_offset)
        out["vc"] = normal_bf16(cshp, SEED_VC + seed_offset)
    if with_grad:
        out["do"] = normal_bf16(shp, SEED_DO + seed_offset)
    if w.qknorm:
        if w.unit_gamma:
            g = np.ones(w.head_dim, dtype=np.float32)
            out["gamma_q"], out["gamma_k"] = g, g.copy()
        else:
            rng = np.random.Generator(np.random.PCG64(SEED_GAMMA + seed_offset))
            out["gamma_q"] = (1.0 + 0.25 * rng.standard_normal(w.head_dim)).astype(np.float32)
            out["gamma_k"] = (1.0 + 0.25 * rng.standard_normal(w.head_dim)).astype(np.float32)
    return out


SEED_FIELD = 9


def add_smooth_field(w: Workload, x: Dict[str, Optional[np.ndarray]], alpha: float = 1.0,
                     n_modes: int = 8, frames: Optional[int] = None,
                     t_offset: int = 0) -> Dict[str, Optional[np.ndarray]]:
    """Structured variant of the i.i.d. inputs: q and k get the same smooth low-frequency
    field over (t, h, w), so neighbouring tokens have similar q and k, as in real video
    latents (i.i.d. N(0,1) tokens have no locality at all).

    Field per head: F(t, y, x) = sum_c cos(2 pi (a_c t/T + b_c y/Hg + c_c x/Wg) + phi_c) W[c, :]
    with integer wave numbers a, b, c in {0, 1, 2}, random phases and W ~ N(0, 1/n_modes) per
    head, so each channel of the field has unit variance; q = q_iid + alpha F, k = k_iid +
    alpha F (bf16 RNE).  Cached frames get the field of their own absolute frames.  Returns a
    new dict; v, dO and the cache values are unchanged.
    """
    rng = np.random.Generator(np.random.PCG64(SEED_FIELD))
    T = w.cached_t + w.t_frames
    waves = rng.integers(0, 3, size=(n_modes, 3)).astype(np.float32)
    waves[0] = (0.0, 1.0, 1.0)  # at least one mode varies in space
    phase = rng.uniform(0.0, 2.0 * np.pi, size=n_modes).astype(np.float32)
    W = (rng.standard_normal((w.heads, n_modes, w.head_dim), dtype=np.float32)
         / np.float32(np.sqrt(n_modes)))

    def field(f0: int, nf: int) -> np.ndarray:
        t = np.arange(f0, f0 + nf, dtype=np.float32)[:, None, None]
        yy = np.arange(w.grid_h, dtype=np.float32)[None, :, None]
        xx = np.arange(w.grid_w, dtype=np.float32)[None, None, :]
        feats = np.stack([np.cos(2 * np.pi * (a * t / T + b * yy / w.grid_h + c * xx / w.grid_w) + p)
                          for (a, b, c), p in zip(waves, phase)], axis=-1)  # [nf, Hg, Wg, C]
        feats = feats.reshape(-1, n_modes)
        wm = np.ascontiguousarray(W.transpose(1, 0, 2).reshape(n_modes, -1))  # [C, H*D]
        return (feats @ wm).reshape(-1, w.heads, w.head_dim)  # [N, H, D]

    out = dict(x)
    cur = field(w.cached_t, w.t_frames)[None] * np.float32(alpha)
    for name in ("q", "k"):
        out[name] = bf16_bits_from_f32(bf16_bits_to_f32(x[name]) + cur)
    if w.cached_t and x.get("kc") is not None:
        out["kc"] = bf16_bits_from_f32(bf16_bits_to_f32(x["kc"]) + field(0, w.cached_t)[None] * np.float32(alpha))
    return out
