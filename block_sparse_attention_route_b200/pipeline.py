"""The BSA call chain on device buffers: prologue -> route -> sparse attention fwd (-> bwd).

``BsaPipeline`` owns the device buffers of one geometry (allocated once with torch) and
issues the C-ABI calls on one stream; it does no arithmetic itself.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import (POOL_MAX, POOL_SUM, ROUTE_POOL_MAX, ROUTE_POOL_SUM, WS_BWD, WS_PROLOGUE_BWD,
               WS_ROUTE, Geometry, Shards, blocked_shape, bsa_attn_bwd, bsa_attn_fwd,
               bsa_block_pool, bsa_blocked_to_raster_sharded, bsa_cache_append, bsa_route_ex,
               bsa_workspace_size, rope3d_qknorm_prologue, rope3d_qknorm_prologue_bwd)


class BsaPipeline:
    """Device buffers + calls for one geometry.

    Inputs are raster bf16 [B, N, H, D] tensors on the device.  ``forward`` fills
    ``self.o`` / ``self.lse`` (blocked), ``self.idx`` / ``self.cnt``; ``backward`` fills
    ``self.dq`` / ``self.dk`` / ``self.dv`` (blocked).
    """

    def __init__(self, g: Geometry, top_r: int, *, rope_theta: float = 10000.0,
                 qknorm: bool = True, eps: float = 1e-6, with_bwd: bool = False,
                 device: str = "cuda"):
        self.g, self.r, self.theta, self.eps, self.qknorm = g, top_r, rope_theta, eps, qknorm
        self.route_flags = 0  # ROUTE_* variant used by forward()
        dev = torch.device(device)
        bf = dict(dtype=torch.bfloat16, device=dev)
        shp = blocked_shape(g)
        self.q = torch.empty(shp, **bf)
        self.k = torch.empty(shp, **bf)
        self.v = torch.empty(shp, **bf)
        self.o = torch.empty(shp, **bf)
        self.lse = torch.empty(shp[:4], dtype=torch.float32, device=dev)
        self.q_pool = torch.empty(shp[:3] + (g.head_dim,), dtype=torch.float32, device=dev)
        self.k_pool = torch.empty_like(self.q_pool)
        self.idx = torch.empty((g.batch, g.heads, g.nbq, top_r), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((g.batch, g.heads, g.nbq), dtype=torch.int32, device=dev)
        self.ws_route = torch.empty(max(bsa_workspace_size(g, top_r, WS_ROUTE), 256),
                                    dtype=torch.uint8, device=dev)
        self.kc = self.vc = self.kc_pool = None
        if g.cached_t:
            cshp = blocked_shape(g, g.cached_t)
            self.kc = torch.empty(cshp, **bf)
            self.vc = torch.empty(cshp, **bf)
            self.kc_pool = torch.empty(cshp[:3] + (g.head_dim,), dtype=torch.float32, device=dev)
            # the cache's keys pooled by a routing variant (sum / max), filled per route call
            self.kc_pool_variant = torch.empty_like(self.kc_pool)
        self.gamma_q = self.gamma_k = None
        self.ws_pro_bwd = None
        if with_bwd:
            self.do = torch.empty(shp, **bf)
            self.dq = torch.empty(shp, **bf)
            self.dk = torch.empty(shp, **bf)
            self.dv = torch.empty(shp, **bf)
            self.ws_bwd = torch.empty(max(bsa_workspace_size(g, top_r, WS_BWD), 256),
                                      dtype=torch.uint8, device=dev)

    def set_gamma(self, gamma_q: Optional[torch.Tensor], gamma_k: Optional[torch.Tensor]):
        self.gamma_q, self.gamma_k = gamma_q, gamma_k

    def load_cache(self, kc_raster: torch.Tensor, vc_raster: torch.Tensor, stream=None):
        """Relayout (and norm/rotate) the cached frames' K/V and their block means, once."""
        g = self.g
        rope3d_qknorm_prologue(g, g.cached_t, 0, None, kc_raster, vc_raster, None,
                               self.gamma_k if self.qknorm else None, self.eps,
                               self.theta, None, self.kc, self.vc, None, self.kc_pool,
                               stream=stream)

    def set_cache(self, kc_blk: torch.Tensor, vc_blk: torch.Tensor, kc_pool: torch.Tensor):
        """Use blocked cache tensors made earlier (e.g. by next_round_cache of the previous
        round) instead of running the prologue on raster cache frames."""
        assert self.kc is not None and kc_blk.shape == self.kc.shape and vc_blk.shape == self.vc.shape
        assert kc_pool.shape == self.kc_pool.shape
        self.kc, self.vc, self.kc_pool = kc_blk, vc_blk, kc_pool

    def next_round_cache(self, stream=None):
        """The cache for the next continuation round: this round's cached blocks followed by
        its current blocks (K, V and the key-block means), as new tensors."""
        g = self.g
        nb = g.nbc + g.nbq
        kc = torch.empty((g.batch, g.heads, nb, g.bs, g.head_dim), dtype=self.k.dtype,
                         device=self.k.device)
        vc = torch.empty_like(kc)
        kp = torch.empty((g.batch, g.heads, nb, g.head_dim), dtype=torch.float32,
                         device=self.k.device)
        bsa_cache_append(g, self.kc, self.vc, self.kc_pool, self.k, self.v, self.k_pool, kc, vc,
                         kp, stream=stream)
        return kc, vc, kp

    def prologue(self, q_raster, k_raster, v_raster, stream=None):
        g = self.g
        rope3d_qknorm_prologue(g, g.t_frames, g.cached_t, q_raster, k_raster, v_raster,
                               self.gamma_q if self.qknorm else None,
                               self.gamma_k if self.qknorm else None, self.eps, self.theta,
                               self.q, self.k, self.v, self.q_pool, self.k_pool, stream=stream)

    def route(self, stream=None, use_pools: bool = True, flags: int = 0):
        """Top-r routing into idx / cnt.  ``flags``: ROUTE_* variants.  A pooling variant pools
        q / k (and the cache's keys) itself instead of using the prologue's block means."""
        kc_pool = self.kc_pool
        pool_mode = POOL_SUM if flags & ROUTE_POOL_SUM else POOL_MAX if flags & ROUTE_POOL_MAX else 0
        if pool_mode:
            use_pools = False
            if self.kc is not None:
                kc_pool = self.kc_pool_variant
                bsa_block_pool(self.g, self.g.cached_t, pool_mode, self.kc, kc_pool, stream=stream)
        bsa_route_ex(self.g, self.r, flags, self.q, self.k, self.q_pool if use_pools else None,
                     self.k_pool if use_pools else None, kc_pool, self.idx, self.cnt,
                     self.ws_route, stream=stream)

    def attn_fwd(self, stream=None):
        bsa_attn_fwd(self.g, self.r, self.q, self.k, self.v, self.kc, self.vc, self.idx,
                     self.cnt, self.o, self.lse, stream=stream)

    def forward(self, q_raster, k_raster, v_raster, stream=None) -> Dict[str, torch.Tensor]:
        self.prologue(q_raster, k_raster, v_raster, stream)
        self.route(stream, flags=self.route_flags)
        self.attn_fwd(stream)
        return {"o": self.o, "lse": self.lse, "idx": self.idx, "cnt": self.cnt}

    def o_to_raster(self, o_raster, stream=None):
        """The blocked output O back in the raster layout [B, T*H*W, heads, D] (pad slots
        dropped): the inverse relayout, with one shard holding every frame."""
        g = self.g
        bsa_blocked_to_raster_sharded(g, g.t_frames, Shards(1, g.t_frames, g.heads, 0), self.o,
                                      [o_raster], stream=stream)

    def load_grad(self, do_raster, stream=None):
        """Relayout the upstream gradient dO (raster) into the blocked layout."""
        g = self.g
        rope3d_qknorm_prologue(g, g.t_frames, 0, None, None, do_raster, None, None, 0.0, 0.0,
                               None, None, self.do, None, None, stream=stream)

    def backward(self, stream=None):
        bsa_attn_bwd(self.g, self.r, self.q, self.k, self.v, self.kc, self.vc, self.o,
                     self.lse, self.do, self.idx, self.cnt, self.dq, self.dk, self.dv,
                     self.ws_bwd, stream=stream)
        return {"dq": self.dq, "dk": self.dk, "dv": self.dv}

    def prologue_backward(self, q_raster, k_raster, dq_raster, dk_raster, dv_raster,
                          dgamma_q=None, dgamma_k=None, stream=None):
        """Gradients of the raster q, k, v (and of the gains) from the blocked dq, dk, dv of
        backward(); q_raster / k_raster are the inputs the forward prologue was given."""
        g = self.g
        if self.ws_pro_bwd is None:
            self.ws_pro_bwd = torch.empty(max(bsa_workspace_size(g, 1, WS_PROLOGUE_BWD), 256),
                                          dtype=torch.uint8, device=self.dq.device)
        gq = self.gamma_q if self.qknorm else None
        gk = self.gamma_k if self.qknorm else None
        rope3d_qknorm_prologue_bwd(g, g.t_frames, g.cached_t, q_raster, k_raster, gq, gk,
                                   self.eps, self.theta, self.dq, self.dk, self.dv, dq_raster,
                                   dk_raster, dv_raster, dgamma_q if gq is not None else None,
                                   dgamma_k if gk is not None else None, self.ws_pro_bwd,
                                   stream=stream)
