"""Sequence-parallel (Ulysses) BSA over the ranks of one node.

Source: "LongCat-Video : Generate 1 minute long AI videos with this model", section "How to
run it" (multi-GPU inference with Ulysses context parallelism) and the Meituan talk, section
2.2 (the sparse attention is trained in parallel).  The raster q, k, v (and O, dO, dq, dk, dv)
of a DiT are split by frames over R ranks; each rank routes and attends a slice of H / R heads
over the whole video.  The two all-to-all exchanges of Ulysses are folded into the library's
relayouts: the sharded prologue reads every rank's frame shard through device pointers of the
peer GPUs (CUDA IPC), and the inverse relayout writes O (or the input gradients) straight into
every rank's shard.  No collective library call carries tensor data; the ranks meet at host
barriers before reading peer shards and after writing them, and sum the gains' gradients (D
floats) with one all-reduce.

This module is host logic only: the plan (who holds which frames and heads), the exchange of
IPC handles, and the order of the library calls.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Dict, List, Optional, Sequence

import torch

from . import (MAX_SHARDS, WS_BWD, WS_PROLOGUE_BWD, WS_ROUTE, Geometry, Shards, blocked_shape,
               bsa_attn_bwd, bsa_attn_fwd, bsa_blocked_to_raster_sharded, bsa_ipc_close,
               bsa_ipc_export, bsa_ipc_import, bsa_route, bsa_workspace_size,
               rope3d_qknorm_prologue_bwd_sharded, rope3d_qknorm_prologue_sharded)


@dataclasses.dataclass(frozen=True)
class UlyssesPlan:
    """Rank `rank` of `world` holds frames [rank * F, (rank + 1) * F) of every raster tensor
    (F = frames / world) for all heads, and computes heads [rank * Hl, (rank + 1) * Hl)
    (Hl = heads / world) over all frames."""
    world: int
    rank: int
    heads: int
    frames: int

    def __post_init__(self):
        if not 1 <= self.world <= MAX_SHARDS:
            raise ValueError(f"world size {self.world} outside 1..{MAX_SHARDS}")
        if not 0 <= self.rank < self.world:
            raise ValueError("rank outside the group")
        if self.heads % self.world or self.frames % self.world:
            raise ValueError("heads and frames must divide evenly over the ranks")

    @property
    def heads_local(self) -> int:
        return self.heads // self.world

    @property
    def head0(self) -> int:
        return self.rank * self.heads_local

    @property
    def shard_frames(self) -> int:
        return self.frames // self.world

    @property
    def frame0(self) -> int:
        return self.rank * self.shard_frames

    def shards(self) -> Shards:
        return Shards(self.world, self.shard_frames, self.heads, self.head0)

    def local_geometry(self, g: Geometry) -> Geometry:
        """The geometry of this rank's attention: all frames, its slice of the heads."""
        return dataclasses.replace(g, heads=self.heads_local)

    def shard_tokens(self, g: Geometry) -> int:
        return self.shard_frames * g.grid_h * g.grid_w


def exchange_pointers(tensors: Dict[str, torch.Tensor], group=None,
                      export: Callable = bsa_ipc_export, import_: Callable = bsa_ipc_import):
    """Every rank passes its own shard tensors (same names on every rank); returns, per name,
    the device pointers of all ranks' shards in rank order (own shard: its local pointer;
    peers': mapped through CUDA IPC) and the list of imported pointers to close later."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    names = sorted(tensors)
    mine = {n: export(tensors[n]) for n in names}
    gathered: List[Optional[dict]] = [None] * dist.get_world_size(group)
    dist.all_gather_object(gathered, mine, group=group)
    table: Dict[str, List[int]] = {n: [] for n in names}
    opened: List[int] = []
    for r, handles in enumerate(gathered):
        if set(handles) != set(names):
            raise RuntimeError(f"rank {r} exported {sorted(handles)}, expected {names}")
        for n in names:
            if r == rank:
                table[n].append(tensors[n].data_ptr())
            else:
                p = import_(handles[n])
                opened.append(p)
                table[n].append(p)
    return table, opened


def close_pointers(opened: Sequence[int], close: Callable = bsa_ipc_close):
    for p in opened:
        close(p)


class UlyssesBsa:
    """One rank's share of sequence-parallel BSA.

    ``ptrs`` maps "q", "k", "v", "o" (and, for the backward, "do", "dq", "dk", "dv") to the R
    device pointers of every rank's raster shard [B, F * grid_h * grid_w, H, D] bf16, in rank
    order: from ``exchange_pointers`` across processes, or the local tensors' pointers when
    all shards live in one process.  ``g`` is the full geometry (all heads, all frames).
    """

    def __init__(self, plan: UlyssesPlan, g: Geometry, top_r: int, ptrs: Dict[str, List[int]],
                 *, rope_theta: float = 10000.0, gamma_q=None, gamma_k=None, eps: float = 1e-6,
                 with_bwd: bool = False, device: str = "cuda"):
        if g.cached_t:
            raise ValueError("sequence-parallel continuation caches are not supported")
        if g.t_frames != plan.frames or g.heads != plan.heads:
            raise ValueError("plan and geometry disagree")
        self.plan, self.g, self.r = plan, g, top_r
        self.gl = plan.local_geometry(g)
        self.sh = plan.shards()
        self.ptrs, self.theta, self.eps = ptrs, rope_theta, eps
        self.gamma_q, self.gamma_k = gamma_q, gamma_k
        dev = torch.device(device)
        bf = dict(dtype=torch.bfloat16, device=dev)
        shp = blocked_shape(self.gl)
        self.q, self.k, self.v, self.o = (torch.empty(shp, **bf) for _ in range(4))
        self.lse = torch.empty(shp[:4], dtype=torch.float32, device=dev)
        self.q_pool = torch.empty(shp[:3] + (g.head_dim,), dtype=torch.float32, device=dev)
        self.k_pool = torch.empty_like(self.q_pool)
        self.idx = torch.empty((g.batch, self.gl.heads, self.gl.nbq, top_r), dtype=torch.int32,
                               device=dev)
        self.cnt = torch.empty((g.batch, self.gl.heads, self.gl.nbq), dtype=torch.int32, device=dev)
        self.ws_route = torch.empty(max(bsa_workspace_size(self.gl, top_r, WS_ROUTE), 256),
                                    dtype=torch.uint8, device=dev)
        if with_bwd:
            self.do, self.dq, self.dk, self.dv = (torch.empty(shp, **bf) for _ in range(4))
            self.ws_bwd = torch.empty(max(bsa_workspace_size(self.gl, top_r, WS_BWD), 256),
                                      dtype=torch.uint8, device=dev)
            self.ws_pro = torch.empty(max(bsa_workspace_size(self.gl, 1, WS_PROLOGUE_BWD), 256),
                                      dtype=torch.uint8, device=dev)
            self.dgamma_q = torch.zeros(g.head_dim, dtype=torch.float32, device=dev)
            self.dgamma_k = torch.zeros_like(self.dgamma_q)

    def forward(self, stream=None):
        """Sequence -> head exchange fused into the prologue, local routing and attention, head
        -> sequence exchange fused into the inverse relayout of O.  Every rank's q, k, v shard
        must be complete before the call (barrier), and O shards are complete on all ranks only
        after every rank's call has finished (barrier)."""
        gl, g, p = self.gl, self.g, self.ptrs
        rope3d_qknorm_prologue_sharded(gl, g.t_frames, 0, self.sh, p["q"], p["k"], p["v"],
                                       self.gamma_q, self.gamma_k, self.eps, self.theta, self.q,
                                       self.k, self.v, self.q_pool, self.k_pool, stream=stream)
        bsa_route(gl, self.r, self.q, self.k, self.q_pool, self.k_pool, None, self.idx, self.cnt,
                  self.ws_route, stream=stream)
        bsa_attn_fwd(gl, self.r, self.q, self.k, self.v, None, None, self.idx, self.cnt, self.o,
                     self.lse, stream=stream)
        bsa_blocked_to_raster_sharded(gl, g.t_frames, self.sh, self.o, p["o"], stream=stream)

    def backward(self, stream=None):
        """dO shards -> local blocked dO (layout-only sharded prologue), attention backward,
        then the prologue backward writing dq, dk, dv into every rank's shards.  The gains'
        gradients are this rank's heads only: sum them over the ranks (all_reduce_gains)."""
        gl, g, p = self.gl, self.g, self.ptrs
        rope3d_qknorm_prologue_sharded(gl, g.t_frames, 0, self.sh, None, None, p["do"], None, None,
                                       0.0, 0.0, None, None, self.do, stream=stream)
        bsa_attn_bwd(gl, self.r, self.q, self.k, self.v, None, None, self.o, self.lse, self.do,
                     self.idx, self.cnt, self.dq, self.dk, self.dv, self.ws_bwd, stream=stream)
        rope3d_qknorm_prologue_bwd_sharded(
            gl, g.t_frames, 0, self.sh, p["q"], p["k"], self.gamma_q, self.gamma_k, self.eps,
            self.theta, self.dq, self.dk, self.dv, p["dq"], p["dk"], p["dv"],
            self.dgamma_q if self.gamma_q is not None else None,
            self.dgamma_k if self.gamma_k is not None else None, self.ws_pro, stream=stream)

    def all_reduce_gains(self, group=None):
        """Sum the gains' gradients over the ranks (the one reduction of the backward)."""
        import torch.distributed as dist
        host = dist.get_backend(group) == "gloo"  # gloo reduces host tensors
        for t, gam in ((self.dgamma_q, self.gamma_q), (self.dgamma_k, self.gamma_k)):
            if gam is None:
                continue
            if host:
                c = t.cpu()
                dist.all_reduce(c, group=group)
                t.copy_(c)
            else:
                dist.all_reduce(t, group=group)


def rank_barrier(group=None):
    """Order cross-rank reads and writes of the shards: this rank's work on its stream is
    done, then every rank has reached the same point."""
    import torch.distributed as dist
    torch.cuda.synchronize()
    dist.barrier(group=group)
