"""Block sparse attention over 3D latent video tokens on B200 (sm_100a).

Thin ctypes binding over ``libbsa.so`` (the C ABI in ``include/bsa.h``).  Functions keep
the C names and only marshal arguments: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  There is no CPU fallback: importing
works without a GPU, but every compute call needs the built library and an sm_100 device.

Build the library with ``python -m block_sparse_attention_route_b200.build``.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from typing import Optional

__all__ = [
    "Geometry", "BsaError", "lib", "bsa_workspace_size", "rope3d_qknorm_prologue", "bsa_route",
    "bsa_attn_fwd", "bsa_attn_bwd", "bsa_device_status", "bsa_error_string", "blocked_shape",
    "bsa_selftest_bounded_wait", "bsa_route_noalloc", "rope3d_qknorm_prologue_bwd",
    "bsa_cache_append", "bsa_route_ex", "bsa_block_pool", "ROUTE_FORCE_SELF",
    "ROUTE_SHARED_HEADS", "ROUTE_POOL_SUM", "ROUTE_POOL_MAX", "POOL_MEAN", "POOL_SUM", "POOL_MAX",
    "Shards", "MAX_SHARDS", "IPC_HANDLE_BYTES", "rope3d_qknorm_prologue_sharded",
    "rope3d_qknorm_prologue_bwd_sharded", "bsa_blocked_to_raster_sharded", "bsa_ipc_export",
    "bsa_ipc_import", "bsa_ipc_close",
    "bsa_kernel_timing", "bsa_kernel_times", "bsa_kernel_time_stats",
    "WS_ROUTE", "WS_FWD", "WS_BWD", "WS_PROLOGUE_BWD",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")
WS_ROUTE, WS_FWD, WS_BWD, WS_PROLOGUE_BWD = 1, 2, 3, 4
ROUTE_FORCE_SELF, ROUTE_SHARED_HEADS, ROUTE_POOL_SUM, ROUTE_POOL_MAX = 1, 2, 4, 8
POOL_MEAN, POOL_SUM, POOL_MAX = 0, 1, 2
STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_CUDA",
          4: "BSA_ERR_TIMEOUT", 5: "BSA_ERR_BAD_INDEX", 6: "BSA_ERR_WORKSPACE"}


class BsaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS.get(code, code)} ({detail})")
        self.code = code


class _Geom(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("t_frames", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("cached_t", ctypes.c_int32), ("blk_t", ctypes.c_int32), ("blk_h", ctypes.c_int32),
                ("blk_w", ctypes.c_int32), ("causal_chunk_t", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("cond_t", ctypes.c_int32)]


MAX_SHARDS, IPC_HANDLE_BYTES = 8, 128


class _Shards(ctypes.Structure):
    _fields_ = [("n_shards", ctypes.c_int32), ("shard_frames", ctypes.c_int32),
                ("heads_total", ctypes.c_int32), ("head0", ctypes.c_int32)]


@dataclasses.dataclass(frozen=True)
class Shards:
    """Mirror of ``bsa_shards_t``: raster tensors split by frames into ``n_shards`` pieces of
    ``shard_frames`` frames with ``heads_total`` heads per row; a call processes heads
    ``head0`` .. ``head0 + g.heads - 1``."""
    n_shards: int
    shard_frames: int
    heads_total: int
    head0: int = 0

    def c(self) -> _Shards:
        return _Shards(self.n_shards, self.shard_frames, self.heads_total, self.head0)


@dataclasses.dataclass(frozen=True)
class Geometry:
    """Mirror of ``bsa_geom_t`` (see include/bsa.h for the meaning of every field)."""
    batch: int
    heads: int
    head_dim: int
    t_frames: int
    grid_h: int
    grid_w: int
    blk: tuple = (4, 4, 8)
    cached_t: int = 0
    causal_chunk_t: int = 0
    softmax_scale: float = 0.0
    cond_t: int = 0

    def c(self) -> _Geom:
        return _Geom(self.batch, self.heads, self.head_dim, self.t_frames, self.grid_h,
                     self.grid_w, self.cached_t, self.blk[0], self.blk[1], self.blk[2],
                     self.causal_chunk_t, float(self.softmax_scale), self.cond_t)

    @property
    def bs(self) -> int:
        return self.blk[0] * self.blk[1] * self.blk[2]

    def n_blocks(self, frames: int) -> int:
        up = lambda x, b: -(-x // b)  # noqa: E731
        return up(frames, self.blk[0]) * up(self.grid_h, self.blk[1]) * up(self.grid_w, self.blk[2])

    @property
    def nbq(self) -> int:
        return self.n_blocks(self.t_frames)

    @property
    def nbc(self) -> int:
        return self.n_blocks(self.cached_t) if self.cached_t else 0

    @property
    def scale(self) -> float:
        return self.softmax_scale or 1.0 / math.sqrt(self.head_dim)

    @classmethod
    def from_workload(cls, w) -> "Geometry":
        return cls(w.batch, w.heads, w.head_dim, w.t_frames, w.grid_h, w.grid_w, tuple(w.blk),
                   w.cached_t, w.chunk_t, cond_t=getattr(w, "cond_t", 0))


def blocked_shape(g: Geometry, frames: Optional[int] = None):
    """Shape [B, H, NB, BS, D] of the blocked layout over ``frames`` (default t_frames)."""
    return (g.batch, g.heads, g.n_blocks(frames or g.t_frames), g.bs, g.head_dim)


_lib = None


def lib() -> ctypes.CDLL:
    """Load libbsa.so; raises if it has not been built (there is no fallback path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m block_sparse_attention_route_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, F, S = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
        G = ctypes.POINTER(_Geom)
        SH = ctypes.POINTER(_Shards)
        sig = {
            "bsa_abi_version": (I32, []),
            "bsa_workspace_size": (S, [G, I32, I32]),
            "rope3d_qknorm_prologue": (I32, [G, I32, I32, P, P, P, P, P, F, F, P, P, P, P, P, P]),
            "rope3d_qknorm_prologue_bwd": (I32, [G, I32, I32, P, P, P, P, F, F, P, P, P, P, P, P,
                                                 P, P, P, S, P]),
            "bsa_route": (I32, [G, I32, P, P, P, P, P, P, P, P, S, P]),
            "bsa_route_ex": (I32, [G, I32, ctypes.c_uint32, P, P, P, P, P, P, P, P, S, P]),
            "bsa_block_pool": (I32, [G, I32, I32, P, P, P]),
            "bsa_attn_fwd": (I32, [G, I32, P, P, P, P, P, P, P, P, P, P]),
            "bsa_attn_bwd": (I32, [G, I32, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P]),
            "bsa_device_status": (I32, [P]),
            "bsa_selftest_bounded_wait": (I32, [I32, P]),
            "bsa_route_noalloc": (I32, [G, I32, P, P, P, P, P, P]),
            "bsa_kernel_timing": (I32, [I32]),
            "bsa_cache_append": (I32, [G, P, P, P, P, P, P, P, P, P, P]),
            "rope3d_qknorm_prologue_sharded": (I32, [G, I32, I32, SH, P, P, P, P, P, F, F, P, P,
                                                     P, P, P, P]),
            "rope3d_qknorm_prologue_bwd_sharded": (I32, [G, I32, I32, SH, P, P, P, P, F, F, P, P,
                                                         P, P, P, P, P, P, P, S, P]),
            "bsa_blocked_to_raster_sharded": (I32, [G, I32, SH, P, P, P]),
            "bsa_ipc_export": (I32, [P, P]),
            "bsa_ipc_import": (I32, [P, ctypes.POINTER(ctypes.c_void_p)]),
            "bsa_ipc_close": (I32, [P]),
            "bsa_kernel_times": (I32, [P, P]),
            "bsa_kernel_time_stats": (I32, [P, P, P, P]),
            "bsa_error_string": (ctypes.c_char_p, [I32]),
            "bsa_last_error_detail": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("tensor arguments must live on the GPU")
    if not t.is_contiguous():
        raise ValueError("tensor arguments must be contiguous")
    return t.data_ptr()


def _nbytes(t) -> int:
    if t is None or isinstance(t, int):
        return 0
    return t.numel() * t.element_size()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return stream if isinstance(stream, int) else stream.cuda_stream


def _check(code: int, where: str):
    if code != 0:
        raise BsaError(code, where, lib().bsa_last_error_detail().decode())


def bsa_error_string(code: int) -> str:
    return lib().bsa_error_string(code).decode()


def bsa_workspace_size(g: Geometry, top_r: int, which: int) -> int:
    return int(lib().bsa_workspace_size(ctypes.byref(g.c()), top_r, which))


def rope3d_qknorm_prologue(g: Geometry, frames: int, t_offset: int, q, k, v, gamma_q, gamma_k,
                           eps: float, rope_theta: float, q_blk, k_blk, v_blk, q_pool=None,
                           k_pool=None, stream=None):
    _check(lib().rope3d_qknorm_prologue(
        ctypes.byref(g.c()), frames, t_offset, _ptr(q), _ptr(k), _ptr(v), _ptr(gamma_q),
        _ptr(gamma_k), eps, rope_theta, _ptr(q_blk), _ptr(k_blk), _ptr(v_blk), _ptr(q_pool),
        _ptr(k_pool), _stream(stream)), "rope3d_qknorm_prologue")


def rope3d_qknorm_prologue_bwd(g: Geometry, frames: int, t_offset: int, q, k, gamma_q, gamma_k,
                               eps: float, rope_theta: float, dq_blk, dk_blk, dv_blk, dq, dk, dv,
                               dgamma_q=None, dgamma_k=None, ws=None, stream=None):
    _check(lib().rope3d_qknorm_prologue_bwd(
        ctypes.byref(g.c()), frames, t_offset, _ptr(q), _ptr(k), _ptr(gamma_q), _ptr(gamma_k),
        eps, rope_theta, _ptr(dq_blk), _ptr(dk_blk), _ptr(dv_blk), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(dgamma_q), _ptr(dgamma_k), _ptr(ws), _nbytes(ws) if ws is not None else 0,
        _stream(stream)), "rope3d_qknorm_prologue_bwd")


def _ptr_array(ts):
    """Host array of device pointers (one per shard), or None."""
    if ts is None:
        return None
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return ctypes.cast(arr, ctypes.c_void_p), arr  # keep `arr` alive for the call


def _arr(x):
    return None if x is None else x[0]


def rope3d_qknorm_prologue_sharded(g: Geometry, frames: int, t_offset: int, sh: Shards,
                                   q_shards, k_shards, v_shards, gamma_q, gamma_k, eps: float,
                                   rope_theta: float, q_blk, k_blk, v_blk, q_pool=None,
                                   k_pool=None, stream=None):
    """The prologue reading raster inputs from frame shards (lists of tensors or pointers)."""
    qa, ka, va = _ptr_array(q_shards), _ptr_array(k_shards), _ptr_array(v_shards)
    _check(lib().rope3d_qknorm_prologue_sharded(
        ctypes.byref(g.c()), frames, t_offset, ctypes.byref(sh.c()), _arr(qa), _arr(ka), _arr(va),
        _ptr(gamma_q), _ptr(gamma_k), eps, rope_theta, _ptr(q_blk), _ptr(k_blk), _ptr(v_blk),
        _ptr(q_pool), _ptr(k_pool), _stream(stream)), "rope3d_qknorm_prologue_sharded")


def rope3d_qknorm_prologue_bwd_sharded(g: Geometry, frames: int, t_offset: int, sh: Shards,
                                       q_shards, k_shards, gamma_q, gamma_k, eps: float,
                                       rope_theta: float, dq_blk, dk_blk, dv_blk, dq_shards,
                                       dk_shards, dv_shards, dgamma_q=None, dgamma_k=None,
                                       ws=None, stream=None):
    qa, ka = _ptr_array(q_shards), _ptr_array(k_shards)
    dqa, dka, dva = _ptr_array(dq_shards), _ptr_array(dk_shards), _ptr_array(dv_shards)
    _check(lib().rope3d_qknorm_prologue_bwd_sharded(
        ctypes.byref(g.c()), frames, t_offset, ctypes.byref(sh.c()), _arr(qa), _arr(ka),
        _ptr(gamma_q), _ptr(gamma_k), eps, rope_theta, _ptr(dq_blk), _ptr(dk_blk), _ptr(dv_blk),
        _arr(dqa), _arr(dka), _arr(dva), _ptr(dgamma_q), _ptr(dgamma_k), _ptr(ws),
        _nbytes(ws) if ws is not None else 0, _stream(stream)), "rope3d_qknorm_prologue_bwd_sharded")


def bsa_blocked_to_raster_sharded(g: Geometry, frames: int, sh: Shards, x_blk, x_shards,
                                  stream=None):
    xa = _ptr_array(x_shards)
    _check(lib().bsa_blocked_to_raster_sharded(
        ctypes.byref(g.c()), frames, ctypes.byref(sh.c()), _ptr(x_blk), _arr(xa), _stream(stream)),
        "bsa_blocked_to_raster_sharded")


def bsa_ipc_export(t) -> bytes:
    """IPC handle (IPC_HANDLE_BYTES bytes) of the device buffer holding tensor / pointer t."""
    buf = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(lib().bsa_ipc_export(_ptr(t), buf), "bsa_ipc_export")
    return buf.raw


def bsa_ipc_import(handle: bytes) -> int:
    """Device pointer (int) mapping another process's buffer; release with bsa_ipc_close."""
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("bad IPC handle length")
    out = ctypes.c_void_p()
    _check(lib().bsa_ipc_import(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES),
                                ctypes.byref(out)), "bsa_ipc_import")
    return int(out.value)


def bsa_ipc_close(ptr: int):
    _check(lib().bsa_ipc_close(ptr), "bsa_ipc_close")


def bsa_cache_append(g: Geometry, kc_blk, vc_blk, kc_pool, k_blk, v_blk, k_pool, kc_new, vc_new,
                     kc_pool_new=None, stream=None):
    _check(lib().bsa_cache_append(
        ctypes.byref(g.c()), _ptr(kc_blk), _ptr(vc_blk), _ptr(kc_pool), _ptr(k_blk), _ptr(v_blk),
        _ptr(k_pool), _ptr(kc_new), _ptr(vc_new), _ptr(kc_pool_new), _stream(stream)),
        "bsa_cache_append")


def bsa_route(g: Geometry, top_r: int, q_blk, k_blk, q_pool, k_pool, kpool_cache, idx, cnt,
              ws=None, stream=None):
    nbytes = _nbytes(ws)
    _check(lib().bsa_route(
        ctypes.byref(g.c()), top_r, _ptr(q_blk), _ptr(k_blk), _ptr(q_pool), _ptr(k_pool),
        _ptr(kpool_cache), _ptr(idx), _ptr(cnt), _ptr(ws), nbytes, _stream(stream)), "bsa_route")


def bsa_route_ex(g: Geometry, top_r: int, flags: int, q_blk, k_blk, q_pool, k_pool, kpool_cache,
                 idx, cnt, ws=None, stream=None):
    nbytes = _nbytes(ws)
    _check(lib().bsa_route_ex(
        ctypes.byref(g.c()), top_r, flags, _ptr(q_blk), _ptr(k_blk), _ptr(q_pool), _ptr(k_pool),
        _ptr(kpool_cache), _ptr(idx), _ptr(cnt), _ptr(ws), nbytes, _stream(stream)),
        "bsa_route_ex")


def bsa_block_pool(g: Geometry, frames: int, mode: int, x_blk, out, stream=None):
    _check(lib().bsa_block_pool(ctypes.byref(g.c()), frames, mode, _ptr(x_blk), _ptr(out),
                                _stream(stream)), "bsa_block_pool")


def bsa_route_noalloc(g: Geometry, top_r: int, q_blk, k_blk, kpool_cache, idx, cnt, stream=None):
    """bsa_route without a workspace (the library's fixed scratch array; see include/bsa.h)."""
    _check(lib().bsa_route_noalloc(
        ctypes.byref(g.c()), top_r, _ptr(q_blk), _ptr(k_blk), _ptr(kpool_cache), _ptr(idx),
        _ptr(cnt), _stream(stream)), "bsa_route_noalloc")


def bsa_attn_fwd(g: Geometry, top_r: int, q_blk, k_blk, v_blk, k_cache_blk, v_cache_blk, idx,
                 cnt, o_blk, lse, stream=None):
    _check(lib().bsa_attn_fwd(
        ctypes.byref(g.c()), top_r, _ptr(q_blk), _ptr(k_blk), _ptr(v_blk), _ptr(k_cache_blk),
        _ptr(v_cache_blk), _ptr(idx), _ptr(cnt), _ptr(o_blk), _ptr(lse), _stream(stream)),
        "bsa_attn_fwd")


def bsa_attn_bwd(g: Geometry, top_r: int, q_blk, k_blk, v_blk, k_cache_blk, v_cache_blk, o_blk,
                 lse, do_blk, idx, cnt, dq_blk, dk_blk, dv_blk, ws, stream=None):
    nbytes = _nbytes(ws)
    _check(lib().bsa_attn_bwd(
        ctypes.byref(g.c()), top_r, _ptr(q_blk), _ptr(k_blk), _ptr(v_blk), _ptr(k_cache_blk),
        _ptr(v_cache_blk), _ptr(o_blk), _ptr(lse), _ptr(do_blk), _ptr(idx), _ptr(cnt),
        _ptr(dq_blk), _ptr(dk_blk), _ptr(dv_blk), _ptr(ws), nbytes, _stream(stream)),
        "bsa_attn_bwd")


def bsa_selftest_bounded_wait(limit_us: int, stream=None):
    _check(lib().bsa_selftest_bounded_wait(limit_us, _stream(stream)), "bsa_selftest_bounded_wait")


TIMED_KERNELS = ("fwd", "bwd_dkdv", "bwd_dq")  # BSA_TIMED_* order


def bsa_kernel_timing(on: bool):
    """Start (True) or stop (False) CUDA-event timing of the attention kernels; either call
    discards what was recorded."""
    _check(lib().bsa_kernel_timing(1 if on else 0), "bsa_kernel_timing")


def bsa_kernel_times() -> dict:
    """Per timed kernel: (launches, total ms) since the last call; waits for the events."""
    n = (ctypes.c_int32 * len(TIMED_KERNELS))()
    ms = (ctypes.c_float * len(TIMED_KERNELS))()
    _check(lib().bsa_kernel_times(ctypes.addressof(n), ctypes.addressof(ms)), "bsa_kernel_times")
    return {k: (int(n[i]), float(ms[i])) for i, k in enumerate(TIMED_KERNELS)}


def bsa_kernel_time_stats() -> dict:
    """Per timed kernel: (launches, total ms, min ms, median ms) since the last call."""
    k_ = len(TIMED_KERNELS)
    n = (ctypes.c_int32 * k_)()
    tot, mn, med = ((ctypes.c_float * k_)() for _ in range(3))
    _check(lib().bsa_kernel_time_stats(ctypes.addressof(n), ctypes.addressof(tot),
                                       ctypes.addressof(mn), ctypes.addressof(med)),
           "bsa_kernel_time_stats")
    return {k: (int(n[i]), float(tot[i]), float(mn[i]), float(med[i]))
            for i, k in enumerate(TIMED_KERNELS)}


def bsa_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status code (0 = OK)."""
    return int(lib().bsa_device_status(_stream(stream)))
