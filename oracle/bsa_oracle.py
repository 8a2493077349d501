"""Plain fp64 CPU oracle for Block Sparse Attention (BSA) over 3D latent video tokens.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.  The
CUDA library never imports it and it imports nothing from the CUDA library.

What it computes, with the page passages each step follows:

* 3D RoPE and RMSNorm + QK-Norm -- "美团LongCat-Video揭秘：13.6B参数长视频生成模型如何终结画面漂移？"
  (xugj520.cn), section 三 "模型架构" (3D RoPE position encoding; RMSNorm + QKNorm); also
  "LongCat-Video : Generate 1 minute long AI videos with this model", section "How it
  handles long videos" (3D attention with RoPE).  Their backward (gradients to the raster
  q, k and the gains) follows from the same definitions; the talk's section 2.2 says the
  module is used for training.
* 3D blocks ("small 3D cubes"), block scores "by similarity", top-r selection --
  "LongCat-Video : Generate 1 minute long AI videos with this model", section "Sparse
  attention"; "LongCat-Video视频生成模型发布 迈出世界模型探索第一步" (youleyou.com), section
  "块稀疏注意力（BSA）" (split 3D tokens into blocks, keep only the top-r key blocks).
* Exact softmax attention over the selected blocks, forward and backward -- same BSA
  sections; the Meituan talk "LongCat-Video 高效長視頻生成探索世界模型的第壹步", section 2.2
  "高效生成" (the module ships forward and backward code for training and inference).
* Block-causal mask and cached conditioning-frame K/V -- the Meituan talk, section 2.1
  ("Block-Causal" attention enabling a cache for continuation); "LongCat-Video : Generate 1
  minute long AI videos with this model", section "The core idea" (KV caching of the fixed
  conditioning frames).  Causal chunks and the two-segment form (conditioning frames attend
  only among themselves) are one segment rule on absolute frames (``Grid``).
* Routing variants the pages leave open -- "LongCat-Video : Generate 1 minute long AI videos
  with this model", section "Sparse attention" (a block keeps its own company plus the
  relevant neighbours): the forced self-block, one selection shared by all heads (scores
  summed over the heads), and sum / channel-max block pooling (``route`` keywords).

Where the pages are silent, this file takes these readings: mean pooling
over valid tokens, unscaled block scores, routing per (batch, head) on post-prologue q/k,
ties broken by lower key-block index, selected lists in ascending block order, RoPE split
(d_t, d_h, d_w) = (D - 4*floor(D/6), 2*floor(D/6), 2*floor(D/6)) with interleaved adjacent
channel pairs, RMSNorm before RoPE, chunk(t) = floor(t / C) on absolute frames, pad keys
excluded, pad queries output 0 with LSE = -inf.

Every array here is float64 unless stated.  Shapes use B batch, N tokens, H heads, D
head dim; raster token order is (t, h, w) row-major over the valid grid.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Tuple

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------------------
# Geometry: the 3D token grid and its block partition
# ----------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Grid:
    """Latent token grid split into 3D blocks (the "3D cubes" of the BSA section).

    ``t_frames`` current frames (query tokens and current key tokens); ``cached_t`` leading
    frames whose keys and values come from a cache (absolute frames 0..cached_t-1, the
    current frames follow at cached_t..); ``blk`` = (bt, bh, bw); ``chunk_t`` = block-causal
    chunk length in frames (0 = no chunks); ``cond_t`` = leading absolute frames of the
    conditioning segment (0 = none).  Block-causal rule (the Meituan talk, section 2.1): a
    frame's segment is 0 inside the conditioning frames and 1 + (frames past them) // chunk_t
    after them (1 when chunk_t = 0); a query block may use a key block whose first frame lies
    in the same or an earlier segment.  So chunk_t alone gives plain causal chunks, cond_t
    alone the two-segment form (conditioning frames see only themselves, the frames being
    generated see everything).
    """
    t_frames: int
    grid_h: int
    grid_w: int
    blk: Tuple[int, int, int]
    cached_t: int = 0
    chunk_t: int = 0
    cond_t: int = 0

    def __post_init__(self):
        bt = self.blk[0]
        if self.cached_t % bt:
            raise ValueError("cached frames must be a whole number of block frames")
        if self.chunk_t and self.chunk_t % bt:
            raise ValueError("causal chunk must be a whole number of block frames")
        if self.cond_t % bt:
            raise ValueError("conditioning frames must be a whole number of block frames")

    @property
    def masked(self) -> bool:
        return bool(self.chunk_t or self.cond_t)

    def frame_segment(self, t: int) -> int:
        if t < self.cond_t:
            return 0
        return 1 + ((t - self.cond_t) // self.chunk_t if self.chunk_t else 0)

    @property
    def nbt(self) -> int:
        return -(-self.t_frames // self.blk[0])

    @property
    def nbh(self) -> int:
        return -(-self.grid_h // self.blk[1])

    @property
    def nbw(self) -> int:
        return -(-self.grid_w // self.blk[2])

    @property
    def bs(self) -> int:
        return self.blk[0] * self.blk[1] * self.blk[2]

    @property
    def nbq(self) -> int:
        """Number of query blocks (blocks over the current frames)."""
        return self.nbt * self.nbh * self.nbw

    @property
    def nbc(self) -> int:
        """Number of cached key blocks (they come first in global key-block order)."""
        return (self.cached_t // self.blk[0]) * self.nbh * self.nbw

    @property
    def nbk(self) -> int:
        return self.nbc + self.nbq

    def block_members(self, frames: int) -> List[List[int]]:
        """Raster token indices of each block of a ``frames`` x grid_h x grid_w grid.

        Blocks are numbered (block-t, block-h, block-w) row-major; within a block the list
        follows (t, h, w) row-major order.  Pad positions are simply absent.
        """
        bt, bh, bw = self.blk
        nbt = -(-frames // bt)
        members: List[List[int]] = [[] for _ in range(nbt * self.nbh * self.nbw)]
        for t in range(frames):
            for h in range(self.grid_h):
                for w in range(self.grid_w):
                    b = ((t // bt) * self.nbh + h // bh) * self.nbw + w // bw
                    members[b].append((t * self.grid_h + h) * self.grid_w + w)
        return members

    def slot_map(self, frames: int) -> np.ndarray:
        """[NB, BS] raster index held by each slot of the padded block layout (-1 = pad).

        A block whose valid extents are (vt, vh, vw) (the last block along an axis may hold
        fewer frames, rows or columns than the block shape) keeps its tokens in its first
        vt*vh*vw slots, row-major over those extents: slot = (lt*vh + lh)*vw + lw with (lt,
        lh, lw) the token's position inside the block; pad slots follow.  A full block is
        plain (lt, lh, lw) row-major.  This is the blocked memory layout the CUDA library
        writes (the pages fix no layout), restated here independently.
        """
        bt, bh, bw = self.blk
        nbt = -(-frames // bt)
        out = -np.ones((nbt * self.nbh * self.nbw, self.bs), dtype=np.int64)
        for t in range(frames):
            vt = min(bt, frames - (t // bt) * bt)
            for h in range(self.grid_h):
                vh = min(bh, self.grid_h - (h // bh) * bh)
                for w in range(self.grid_w):
                    vw = min(bw, self.grid_w - (w // bw) * bw)
                    b = ((t // bt) * self.nbh + h // bh) * self.nbw + w // bw
                    s = ((t % bt) * vh + h % bh) * vw + w % bw
                    assert s < vt * vh * vw
                    out[b, s] = (t * self.grid_h + h) * self.grid_w + w
        return out

    def query_block_chunk(self, i: int) -> int:
        """Mask segment of query block i (of its first absolute frame)."""
        t0 = self.cached_t + (i // (self.nbh * self.nbw)) * self.blk[0]
        return self.frame_segment(t0)

    def key_block_chunk(self, j: int) -> int:
        """Mask segment of global key block j (cached blocks first)."""
        per_t = self.nbh * self.nbw
        if j < self.nbc:
            t0 = (j // per_t) * self.blk[0]
        else:
            t0 = self.cached_t + ((j - self.nbc) // per_t) * self.blk[0]
        return self.frame_segment(t0)


# ----------------------------------------------------------------------------------------
# Prologue: RMSNorm + QK-Norm, then 3D RoPE
# ----------------------------------------------------------------------------------------
def rope_split(d: int) -> Tuple[int, int, int]:
    """Channel widths (d_t, d_h, d_w) of the three rotary axes (all even, summing to D)."""
    dh = 2 * (d // 6)
    return d - 2 * dh, dh, dh


def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """y = x / sqrt(mean(x^2) + eps) * gamma over the last axis (per token and head)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def rope_angles(pos: np.ndarray, width: int, theta: float) -> np.ndarray:
    """Angles [len(pos), width/2]: pair i of an axis of ``width`` channels turns by
    pos * theta^(-2i/width)."""
    i = np.arange(width // 2, dtype=np.float64)
    inv = np.power(float(theta), -2.0 * i / width)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]


def rope3d(x: np.ndarray, t_pos: np.ndarray, h_pos: np.ndarray, w_pos: np.ndarray,
           theta: float) -> np.ndarray:
    """Rotate adjacent channel pairs (2p, 2p+1) of x [..., N, H, D] by 3D positions.

    Channels [0, d_t) follow the frame index, [d_t, d_t+d_h) the row, the rest the column.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    dt, dh, dw = rope_split(d)
    ang = np.concatenate([rope_angles(t_pos, dt, theta), rope_angles(h_pos, dh, theta),
                          rope_angles(w_pos, dw, theta)], axis=1)  # [N, D/2]
    c = np.cos(ang)[:, None, :]  # broadcast over heads
    s = np.sin(ang)[:, None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = xe * c - xo * s
    y[..., 1::2] = xe * s + xo * c
    return y


def grid_positions(frames: int, grid_h: int, grid_w: int, t_offset: int = 0):
    """(t, h, w) positions of the raster tokens; t is the absolute latent frame."""
    t, h, w = np.meshgrid(np.arange(frames), np.arange(grid_h), np.arange(grid_w),
                          indexing="ij")
    return (t.reshape(-1) + t_offset).astype(np.float64), h.reshape(-1).astype(np.float64), \
        w.reshape(-1).astype(np.float64)


def prologue(x: np.ndarray, frames: int, grid_h: int, grid_w: int, *,
             gamma: Optional[np.ndarray], eps: float = 1e-6, theta: float = 0.0,
             t_offset: int = 0) -> np.ndarray:
    """Per (token, head): RMSNorm over D with gain ``gamma`` (skipped when None), then 3D
    RoPE (skipped when theta == 0).  x is raster [B, N, H, D]; returns fp64, same shape."""
    y = np.asarray(x, dtype=np.float64)
    if gamma is not None:
        y = rms_norm(y, gamma, eps)
    if theta:
        t, h, w = grid_positions(frames, grid_h, grid_w, t_offset)
        y = rope3d(y, t, h, w, theta)
    return y


def rope3d_transpose(dz: np.ndarray, t_pos: np.ndarray, h_pos: np.ndarray, w_pos: np.ndarray,
                     theta: float) -> np.ndarray:
    """Gradient of rope3d with respect to its input: each pair was turned by R(a), so the
    upstream gradient is turned back by R(a)^T (pair (e, o): e' = e cos a + o sin a,
    o' = -e sin a + o cos a), with the same angles as the forward."""
    dz = np.asarray(dz, dtype=np.float64)
    d = dz.shape[-1]
    dt, dh, dw = rope_split(d)
    ang = np.concatenate([rope_angles(t_pos, dt, theta), rope_angles(h_pos, dh, theta),
                          rope_angles(w_pos, dw, theta)], axis=1)
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    ze, zo = dz[..., 0::2], dz[..., 1::2]
    dy = np.empty_like(dz)
    dy[..., 0::2] = ze * c + zo * s
    dy[..., 1::2] = -ze * s + zo * c
    return dy


def rms_norm_bwd(dy: np.ndarray, x: np.ndarray, gamma: np.ndarray, eps: float):
    """Gradients of y = x / r * gamma, r = sqrt(mean(x^2) + eps), over the last axis.

    With xh = x / r: d gamma = sum over every leading index of dy * xh; d xh = dy * gamma;
    dx = (d xh - xh * mean(d xh * xh)) / r (r depends on x through mean(x^2)).
    Returns (dx, dgamma)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    gamma = np.asarray(gamma, dtype=np.float64)
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    xh = x / r
    dgamma = np.sum((dy * xh).reshape(-1, x.shape[-1]), axis=0)
    dxh = dy * gamma
    dx = (dxh - xh * np.mean(dxh * xh, axis=-1, keepdims=True)) / r
    return dx, dgamma


def prologue_bwd(dz: np.ndarray, x: np.ndarray, frames: int, grid_h: int, grid_w: int, *,
                 gamma: Optional[np.ndarray], eps: float = 1e-6, theta: float = 0.0,
                 t_offset: int = 0):
    """Backward of ``prologue``: dz is the gradient of its output (raster [B, N, H, D]), x its
    raster input.  The steps of the forward are undone in reverse order: RoPE (turn back by
    the transposed rotation), then RMSNorm.  Returns (dx, dgamma); dgamma is None when the
    forward had no gain."""
    dy = np.asarray(dz, dtype=np.float64)
    if theta:
        t, h, w = grid_positions(frames, grid_h, grid_w, t_offset)
        dy = rope3d_transpose(dy, t, h, w, theta)
    if gamma is None:
        return dy, None
    return rms_norm_bwd(dy, x, gamma, eps)


# ----------------------------------------------------------------------------------------
# Routing: block pooling, block scores, top-r
# ----------------------------------------------------------------------------------------
def block_means(x: np.ndarray, members: List[List[int]]) -> np.ndarray:
    """Mean over the valid tokens of each block: x raster [B, N, H, D] -> [B, H, NB, D]."""
    return block_pool(x, members, "mean")


def block_pool(x: np.ndarray, members: List[List[int]], mode: str = "mean") -> np.ndarray:
    """One vector per block from its valid tokens: x raster [B, N, H, D] -> [B, H, NB, D].

    ``mean`` is the routing's default reading of "blocks chosen by similarity"; ``sum`` and
    ``max`` (channel-wise maximum) are the pooling variants the pages leave open.
    """
    b_, _, h_, d_ = x.shape
    out = np.zeros((b_, h_, len(members), d_), dtype=np.float64)
    for j, idx in enumerate(members):
        if not idx:
            continue
        tok = np.asarray(x[:, idx], dtype=np.float64)  # [B, n_j, H, D]
        if mode == "mean":
            out[:, :, j, :] = tok.mean(axis=1)
        elif mode == "sum":
            out[:, :, j, :] = tok.sum(axis=1)
        elif mode == "max":
            out[:, :, j, :] = tok.max(axis=1)
        else:
            raise ValueError(mode)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray, grid: Grid,
                 key_counts: Optional[List[int]] = None) -> np.ndarray:
    """s[b, h, i, j] = qbar_i . kbar_j (unscaled), -inf where the block-causal rule forbids
    key block j for query block i or key block j holds no valid token."""
    s = np.einsum("bhid,bhjd->bhij", qbar, kbar)
    if grid.masked:
        allowed = np.array([[grid.key_block_chunk(j) <= grid.query_block_chunk(i)
                             for j in range(grid.nbk)] for i in range(grid.nbq)])
        s = np.where(allowed[None, None], s, NEG_INF)
    if key_counts is not None:
        empty = np.array([c == 0 for c in key_counts])
        s = np.where(empty[None, None, None, :], NEG_INF, s)
    return s


def select_top_r(s: np.ndarray, r: int) -> Tuple[np.ndarray, np.ndarray]:
    """Per row: the r largest finite scores, ties to the lower key-block index.

    Returns idx [..., r] int32 listing the chosen blocks in ascending order with -1 padding,
    and cnt [...] = min(r, number of finite scores).
    """
    lead = s.shape[:-1]
    nb = s.shape[-1]
    flat = s.reshape(-1, nb)
    idx = -np.ones((flat.shape[0], r), dtype=np.int32)
    cnt = np.zeros(flat.shape[0], dtype=np.int32)
    cols = np.arange(nb)
    for row in range(flat.shape[0]):
        v = flat[row]
        finite = np.isfinite(v)
        order = np.lexsort((cols, -np.where(finite, v, 0.0)))  # primary: score desc
        order = [j for j in order if finite[j]][:r]
        chosen = np.sort(np.asarray(order, dtype=np.int64))
        idx[row, :len(chosen)] = chosen
        cnt[row] = len(chosen)
    return idx.reshape(lead + (r,)), cnt.reshape(lead)


def select_with_self(s: np.ndarray, r: int, nbc: int) -> Tuple[np.ndarray, np.ndarray]:
    """Forced self-block variant: query block i always keeps its own key block nbc + i,
    and the other r - 1 places go to the best of the remaining blocks (the top-r rule with
    ties to the lower index).  s is [..., NBq, NBk]; same outputs as ``select_top_r``."""
    nbq, nb = s.shape[-2], s.shape[-1]
    idx = -np.ones(s.shape[:-1] + (r,), dtype=np.int32)
    cnt = np.zeros(s.shape[:-1], dtype=np.int32)
    for lead in np.ndindex(s.shape[:-2]):
        for i in range(nbq):
            own = nbc + i
            rest = s[lead + (i,)].copy()
            rest[own] = NEG_INF
            others, n_o = select_top_r(rest[None], r - 1) if r > 1 else (np.zeros((1, 0), np.int32), [0])
            chosen = np.sort(np.concatenate([[own], others[0, :n_o[0]]]))
            idx[lead + (i,)][:len(chosen)] = chosen
            cnt[lead + (i,)] = len(chosen)
    return idx, cnt


def route(q: np.ndarray, k: np.ndarray, grid: Grid, r: int,
          k_cache: Optional[np.ndarray] = None, *, pool: str = "mean",
          force_self: bool = False, shared_heads: bool = False):
    """Block-pooled q.k routing: returns (idx [B,H,NBq,r], cnt [B,H,NBq], scores).

    Variants: ``pool`` = mean | sum | max block pooling; ``force_self`` always keeps a query
    block's own key block; ``shared_heads`` ranks key blocks by the score summed over the
    heads, s_ij = sum_h qbar_hi . kbar_hj, and gives every head that one selection (the
    returned scores are then [B, 1, NBq, NBk]).
    """
    qm = grid.block_members(grid.t_frames)
    qbar = block_pool(q, qm, pool)
    kbar = block_pool(k, qm, pool)
    counts = [len(m) for m in qm]
    if grid.nbc:
        cm = grid.block_members(grid.cached_t)
        kbar = np.concatenate([block_pool(k_cache, cm, pool), kbar], axis=2)
        counts = [len(m) for m in cm] + counts
    s = block_scores(qbar, kbar, grid, counts)
    if shared_heads:
        s = s.sum(axis=1, keepdims=True)
    if force_self:
        idx, cnt = select_with_self(s, r, grid.nbc)
    else:
        idx, cnt = select_top_r(s, r)
    if shared_heads:
        h_ = q.shape[2]
        idx = np.repeat(idx, h_, axis=1)
        cnt = np.repeat(cnt, h_, axis=1)
    return idx, cnt, s


# ----------------------------------------------------------------------------------------
# Exact softmax attention over the selected blocks, forward and backward
# ----------------------------------------------------------------------------------------
def _key_tokens(grid: Grid, sel: np.ndarray, cur_members, cache_members):
    """Token lists (source, raster index) for an ascending list of global key blocks."""
    toks = []
    for j in sel:
        if j < 0:
            continue
        if j < grid.nbc:
            toks.extend(("c", t) for t in cache_members[j])
        else:
            toks.extend(("k", t) for t in cur_members[j - grid.nbc])
    return toks


def _gather(arr_cur, arr_cache, toks, b, h):
    rows = [arr_cur[b, t, h] if src == "k" else arr_cache[b, t, h] for src, t in toks]
    if not rows:
        return np.zeros((0, arr_cur.shape[-1]))
    return np.asarray(rows, dtype=np.float64)


def attend(q, k, v, idx, grid: Grid, scale: float, k_cache=None, v_cache=None,
           return_probs: bool = False, query_blocks: Optional[List[Tuple[int, int, int]]] = None):
    """O = softmax(q k^T * scale) v over the tokens of the selected key blocks.

    q, k, v raster [B, N, H, D] (current frames), k_cache / v_cache raster over the cached
    frames.  idx [B, H, NBq, r] global key-block ids (-1 = unused).  Returns O raster
    [B, N, H, D] and LSE [B, N, H] (natural log); queries of blocks not evaluated keep
    O = 0 and LSE = nan.  ``query_blocks`` restricts the work to (b, h, i) triples.
    With ``return_probs`` also returns {(b, h, i): P} where P is [n_i, n_keys] over the
    selected blocks' key tokens in ascending block order.
    """
    cur = grid.block_members(grid.t_frames)
    cache = grid.block_members(grid.cached_t) if grid.nbc else []
    B, N, H, D = q.shape
    o = np.zeros((B, N, H, D))
    lse = np.full((B, N, H), np.nan)
    probs = {}
    todo = query_blocks if query_blocks is not None else \
        [(b, h, i) for b in range(B) for h in range(H) for i in range(grid.nbq)]
    for b, h, i in todo:
        qi = cur[i]
        if not qi:
            continue
        toks = _key_tokens(grid, idx[b, h, i], cur, cache)
        qm = np.asarray(q[b, qi, h], dtype=np.float64)
        if not toks:  # nothing selected: output 0, LSE -inf
            lse[b, qi, h] = NEG_INF
            continue
        km = _gather(k, k_cache, toks, b, h)
        vm = _gather(v, v_cache, toks, b, h)
        logits = qm @ km.T * scale
        m = logits.max(axis=1, keepdims=True)
        e = np.exp(logits - m)
        l_ = e.sum(axis=1, keepdims=True)
        p = e / l_
        o[b, qi, h] = p @ vm
        lse[b, qi, h] = (m + np.log(l_))[:, 0]
        if return_probs:
            probs[(b, h, i)] = p
    if return_probs:
        return o, lse, probs
    return o, lse


def attend_bwd(q, k, v, do, idx, grid: Grid, scale: float, k_cache=None, v_cache=None,
               query_blocks: Optional[List[Tuple[int, int, int]]] = None):
    """Gradients of sum(dO * O) for O = attend(...): closed form per query block.

    With P the softmax over the selected key tokens and dP = dO V^T:
      dS = P * (dP - rowsum(dO * O)),  dQ = scale * dS K,  dK += scale * dS^T Q,  dV += P^T dO.
    Gradients reach current keys/values only (cached ones are constants).  Returns raster
    dq, dk, dv [B, N, H, D].

    ``query_blocks`` restricts the work to (b, h, i) triples: dQ of those blocks is then
    complete, and dK / dV of a key block are complete when every query block that selected it
    is listed (the rest of dK / dV holds partial sums).
    """
    cur = grid.block_members(grid.t_frames)
    cache = grid.block_members(grid.cached_t) if grid.nbc else []
    B, N, H, D = q.shape
    dq = np.zeros((B, N, H, D))
    dk = np.zeros((B, N, H, D))
    dv = np.zeros((B, N, H, D))
    todo = query_blocks if query_blocks is not None else \
        [(b, h, i) for b in range(B) for h in range(H) for i in range(grid.nbq)]
    for b, h, i in todo:
        qi = cur[i]
        toks = _key_tokens(grid, idx[b, h, i], cur, cache)
        if not qi or not toks:
            continue
        qm = np.asarray(q[b, qi, h], dtype=np.float64)
        km = _gather(k, k_cache, toks, b, h)
        vm = _gather(v, v_cache, toks, b, h)
        dom = np.asarray(do[b, qi, h], dtype=np.float64)
        logits = qm @ km.T * scale
        e = np.exp(logits - logits.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)
        om = p @ vm
        dp = dom @ vm.T
        delta = np.sum(dom * om, axis=1, keepdims=True)
        ds = p * (dp - delta)
        dq[b, qi, h] = scale * ds @ km
        dkm = scale * ds.T @ qm
        dvm = p.T @ dom
        # scatter-add into the current keys' rows (each key token occurs once per list)
        rows = [row for row, (src, _) in enumerate(toks) if src == "k"]
        dst = [t for src, t in toks if src == "k"]
        dk[b, dst, h] += dkm[rows]
        dv[b, dst, h] += dvm[rows]
    return dq, dk, dv


def dense_attention(q, k, v, scale: float):
    """Plain full softmax attention per (batch, head) over all tokens (no blocks)."""
    B, N, H, D = q.shape
    o = np.zeros((B, N, H, D))
    lse = np.zeros((B, N, H))
    for b in range(B):
        for h in range(H):
            logits = np.asarray(q[b, :, h], np.float64) @ np.asarray(k[b, :, h], np.float64).T * scale
            m = logits.max(axis=1, keepdims=True)
            e = np.exp(logits - m)
            l_ = e.sum(axis=1, keepdims=True)
            o[b, :, h] = (e / l_) @ np.asarray(v[b, :, h], np.float64)
            lse[b, :, h] = (m + np.log(l_))[:, 0]
    return o, lse


def near_tie_ok(gpu_sel, ref_sel, scores_row, tau_rel: float = 1e-4) -> bool:
    """Route parity rule for one query block: the two selections may differ only in blocks
    whose score lies within ``tau_rel`` (relative) of the oracle's r-th (threshold) score."""
    g, o = set(int(j) for j in gpu_sel if j >= 0), set(int(j) for j in ref_sel if j >= 0)
    if len(g) != len(o):
        return False
    if g == o:
        return True
    finite = [scores_row[j] for j in o]
    tau = min(finite)
    for j in g ^ o:
        sj = scores_row[j]
        if not math.isfinite(sj):
            return False
        if abs(sj - tau) > tau_rel * max(abs(sj), abs(tau)):
            return False
    return True
