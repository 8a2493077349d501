"""Helpers shared by the GPU tests: bf16 transfer and blocked <-> raster layout via the
oracle's own slot map (so the layout itself is checked against an independent restatement)."""
import numpy as np

import oracle
from synth import bf16_bits_to_f64


def grid_of(w):
    return oracle.Grid(w.t_frames, w.grid_h, w.grid_w, w.blk, w.cached_t, w.chunk_t, w.cond_t)


def to_dev(bits, device="cuda"):
    import torch
    if bits is None:
        return None
    if bits.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(bits)).to(device)


def bf16_dev_to_f64(t):
    import torch
    return bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def blocked_to_raster(blk, slot_map):
    """[B, H, NB, BS, D] -> raster [B, N, H, D] (pad slots dropped)."""
    B, H, NB, BS, D = blk.shape
    valid = slot_map >= 0
    n = int(valid.sum())
    out = np.zeros((B, n, H, D), dtype=blk.dtype)
    bi, si = np.nonzero(valid)
    out[:, slot_map[bi, si]] = blk[:, :, bi, si, :].transpose(0, 2, 1, 3)
    return out


def pad_slots(slot_map):
    return np.nonzero(slot_map < 0)


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (for |x| >= 2^-126)."""
    ax = np.maximum(np.abs(x), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)
