/*
 * bsa.h -- C ABI of the B200 (sm_100a) block sparse attention library (libbsa.so).
 *
 * Block Sparse Attention (BSA) over 3D latent video tokens: the token grid (latent frames x
 * rows x columns) is split into 3D blocks; every query block scores every key block with
 * block-pooled q.k, keeps its top-r key blocks, and exact softmax attention runs over the
 * selected blocks only, with an optional block-causal mask and cached conditioning-frame
 * keys/values.  Sources (web pages describing the LongCat-Video model):
 *   - "LongCat-Video : Generate 1 minute long AI videos with this model", section "Sparse
 *     attention" (small 3D cubes, each looks at the few most relevant ones, chosen by
 *     similarity) and section "The core idea" (KV caching of conditioning frames);
 *   - "LongCat-Video视频生成模型发布 迈出世界模型探索第一步", section 块稀疏注意力（BSA）
 *     (split the 3D tokens into blocks, keep only the top-r key blocks);
 *   - "美团LongCat-Video揭秘：13.6B参数长视频生成模型如何终结画面漂移？", section 三 模型架构
 *     (3D RoPE; RMSNorm + QKNorm);
 *   - "LongCat-Video 高效長視頻生成探索世界模型的第壹步", section 2.1 (Block-Causal
 *     attention enabling a cache for continuation) and 2.2 (the sparse attention module
 *     ships forward and backward code).
 *
 * LAYOUTS (all tensors contiguous, row-major, device memory unless stated)
 *   raster  : bf16 [B, N, H, D], N = frames * grid_h * grid_w tokens ordered (t, h, w).
 *   blocked : bf16 [B, H, NB, BS, D].  The grid is padded up to whole blocks; blocks are
 *             numbered (block-t, block-h, block-w) row-major.  Of the BS = blk_t*blk_h*blk_w
 *             slots of a block with valid extents (vt, vh, vw) (the last block along an
 *             axis may hold fewer frames, rows or columns than the block shape), the first
 *             n = vt*vh*vw hold its tokens, row-major over those extents: slot
 *             (local t * vh + local h) * vw + local w.  A full block is therefore plain
 *             (local t, local h, local w) row-major.  Pad slots (>= n) follow and hold zeros
 *             (written by the prologue, written as zeros in O/dQ/dK/dV).  The valid prefix
 *             lets the attention kernels shrink a partial block's tiles.
 *   pooled  : fp32 [B, H, NB, D], mean over the valid (non-pad) tokens of each block.
 *   idx     : int32 [B, H, NBq, top_r], selected global key-block ids in ascending order,
 *             -1 after the first cnt entries.  cnt: int32 [B, H, NBq].
 *   lse     : fp32 [B, H, NBq, BS], natural-log log-sum-exp of the scaled logits of each
 *             query slot; -inf for pad slots.
 *   Query blocks cover the current frames (NBq blocks).  Key blocks are numbered globally:
 *   first the NBc blocks of the cached frames (read from the *_cache tensors, blocked over
 *   cached_t frames), then the NBq blocks of the current frames.
 *
 * OWNERSHIP AND ORDERING
 *   The caller allocates every buffer; the library allocates no device memory per call.
 *   Scratch memory is the caller's workspace (see bsa_workspace_size).  Every call enqueues
 *   work on `stream` and returns without waiting.  Argument errors are returned before
 *   anything is enqueued.  Device-side failures (a bounded wait that ran out, an index out
 *   of range) set a per-device status word that bsa_device_status() reports; kernels never
 *   trap.  Devices other than sm_100 return BSA_ERR_UNSUPPORTED; there is no fallback.
 */
#ifndef BSA_H_
#define BSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSA_ABI_VERSION 2

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

typedef struct CUstream_st* bsa_stream_t; /* same handle as cudaStream_t; NULL = legacy default stream */

typedef enum bsa_status {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,  /* bad pointer, size, shape or alignment; nothing was enqueued */
  BSA_ERR_UNSUPPORTED = 2,  /* device is not sm_100, or a shape outside the supported set */
  BSA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  BSA_ERR_TIMEOUT = 4,      /* a kernel's bounded wait ran out (reported by bsa_device_status) */
  BSA_ERR_BAD_INDEX = 5,    /* idx/cnt held a value out of range (reported by bsa_device_status) */
  BSA_ERR_WORKSPACE = 6     /* workspace pointer NULL/misaligned or smaller than required */
} bsa_status_t;

/* Geometry of one problem.  Supported: head_dim in {64, 128}; blk_t*blk_h*blk_w in {32, 128}
 * (the backward, bsa_attn_bwd, takes 128 only); cached_t, causal_chunk_t and cond_t multiples
 * of blk_t. */
typedef struct bsa_geom {
  int32_t batch;          /* B */
  int32_t heads;          /* H */
  int32_t head_dim;       /* D */
  int32_t t_frames;       /* current latent frames (query tokens and current key tokens) */
  int32_t grid_h;         /* latent rows (valid, before padding) */
  int32_t grid_w;         /* latent columns (valid, before padding) */
  int32_t cached_t;       /* leading latent frames whose K/V come from the cache (0 = none);
                             current frame f sits at absolute frame cached_t + f */
  int32_t blk_t, blk_h, blk_w; /* 3D block shape */
  int32_t causal_chunk_t; /* C: 0 = no causal chunks */
  float softmax_scale;    /* logits = q.k * scale; 0 selects 1/sqrt(head_dim) */
  int32_t cond_t;         /* leading absolute frames of the conditioning segment (0 = none) */
} bsa_geom_t;
/* Block-causal mask (applied by the routing): with t0 the first absolute frame of a block and
 * seg(t) = 0 for t < cond_t, else 1 + (C ? floor((t - cond_t) / C) : 0), key block j is allowed
 * for query block i iff seg(t0(j)) <= seg(t0(i)).  cond_t = 0 gives plain chunks
 * floor(t/C); C = 0 with cond_t > 0 gives the two-segment form of the continuation task
 * (conditioning frames attend only among themselves, the frames to generate attend to all;
 * "LongCat-Video 高效長視頻生成探索世界模型的第壹步", section 2.1, Block-Causal attention);
 * both 0: no mask.  cond_t must be a multiple of blk_t. */

enum { BSA_WS_ROUTE = 1, BSA_WS_FWD = 2, BSA_WS_BWD = 3, BSA_WS_PROLOGUE_BWD = 4 };

/* ABI version of the loaded library (BSA_ABI_VERSION). */
BSA_API int32_t bsa_abi_version(void);

/* Bytes of workspace `which` (BSA_WS_*) needs for this geometry; 0 on invalid arguments.
 * Workspace must be 256-byte aligned.  ROUTE: pooled q/k means.  FWD: none (returns 0).
 * BWD: per query row -Delta (Delta = rowsum(dO*O)) and -LSE*log2(e), the key-block ->
 * query-block index and a work counter of the dK/dV pass.  PROLOGUE_BWD: fp32 partial sums of
 * d gamma_q and d gamma_k, one D-row per CTA of the prologue backward over g->t_frames frames
 * (top_r is ignored). */
BSA_API size_t bsa_workspace_size(const bsa_geom_t* g, int32_t top_r, int32_t which);

/* Fused QK-RMSNorm + 3D RoPE prologue and raster -> blocked relayout.
 * Source: "美团LongCat-Video揭秘…", section 三 模型架构 (3D RoPE; RMSNorm + QKNorm).
 * Processes `frames` frames of the (grid_h, grid_w) grid of g (pass g->t_frames for the
 * current tokens, g->cached_t for a cache).  For q and k, per (token, head):
 *   y = x / sqrt(mean_d(x^2) + eps) * gamma      (skipped when gamma is NULL)
 *   then 3D RoPE when rope_theta > 0: channels [0,d_t) turn with the absolute frame
 *   (t_offset + t), [d_t, d_t+d_h) with the row, [d_t+d_h, D) with the column, where
 *   d_h = d_w = 2*floor(D/6) and d_t = D - 2*d_h; the adjacent pair (2p, 2p+1) of an axis
 *   of width d_a turns by pos * rope_theta^(-2i/d_a), i = the pair's index in that axis.
 * v is relaid out only (any tensor that needs the layout alone, e.g. dO, can go here).
 * Each of q/k/v may be NULL (then its output must be NULL too).  q_pool / k_pool (nullable)
 * receive the fp32 block means of the bf16-rounded q / k outputs.  Arithmetic in fp32,
 * outputs rounded to bf16 (round to nearest even).  Raster inputs: bf16 [B, frames*gh*gw,
 * H, D]; outputs blocked over `frames` (pad slots zero).  gamma: fp32 [D] device arrays. */
BSA_API bsa_status_t rope3d_qknorm_prologue(const bsa_geom_t* g, int32_t frames, int32_t t_offset,
                                    const void* q_raster, const void* k_raster,
                                    const void* v_raster, const float* gamma_q,
                                    const float* gamma_k, float eps, float rope_theta,
                                    void* q_blk, void* k_blk, void* v_blk, float* q_pool,
                                    float* k_pool, bsa_stream_t stream);

/* Continuation: the cache for the next round.  Source: "LongCat-Video 高效長視頻生成探索世界
 * 模型的第壹步", section 2.1 (Block-Causal attention makes produced frames cacheable), and
 * "LongCat-Video : Generate 1 minute long AI videos with this model", section "The core idea".
 * For geometry g of the round just run (cached_t cached frames, t_frames current frames,
 * t_frames a multiple of blk_t), writes per (b, h) the old cache's NBc blocks followed by the
 * current NBq blocks: kc_new / vc_new bf16 [B, H, NBc + NBq, BS, D] from kc_blk / vc_blk
 * (NULL when cached_t == 0) and the current k_blk / v_blk; kc_pool_new fp32 [B, H, NBc + NBq, D]
 * likewise from kc_pool and k_pool (all three NULL to skip the means).  The result is the
 * cache of a geometry with cached_t + t_frames cached frames.  Keys carry absolute-frame RoPE,
 * so nothing is recomputed.  The caller owns every buffer; the outputs must not overlap the
 * inputs. */
BSA_API bsa_status_t bsa_cache_append(const bsa_geom_t* g, const void* kc_blk, const void* vc_blk,
                                      const float* kc_pool, const void* k_blk, const void* v_blk,
                                      const float* k_pool, void* kc_new, void* vc_new,
                                      float* kc_pool_new, bsa_stream_t stream);

/* Backward of rope3d_qknorm_prologue over the same `frames`, t_offset, gamma, eps and
 * rope_theta.  Same source; the talk "LongCat-Video 高效長視頻生成探索世界模型的第壹步",
 * section 2.2, has the sparse-attention module trained, which needs these gradients.
 * Given dq_blk / dk_blk / dv_blk, the gradients of the blocked outputs (bf16, pad slots
 * ignored), writes the gradients of the raster inputs dq / dk / dv (bf16 [B, frames*gh*gw,
 * H, D]) and, for q / k processed with a gain, dgamma_q / dgamma_k (fp32 [D], overwritten).
 * Per (token, head): dy = RoPE^T(dz) (each pair turned back by its forward angle); with a
 * gain, xh = x / r, r = sqrt(mean_d(x^2) + eps), dgamma += dy * xh (summed over tokens and
 * heads), dx = (dy*gamma - xh * mean_d(dy*gamma*xh)) / r; without one dx = dy.  v: inverse
 * relayout.  q / k (the forward's raster inputs) are needed where a gain is given.  Each of
 * dq_blk / dk_blk / dv_blk may be NULL (then its output must be NULL too).  ws: 256-byte
 * aligned, bsa_workspace_size(g, 1, BSA_WS_PROLOGUE_BWD) bytes when a gain is given, else
 * may be NULL.  dgamma is reduced in a fixed order (deterministic). */
BSA_API bsa_status_t rope3d_qknorm_prologue_bwd(const bsa_geom_t* g, int32_t frames, int32_t t_offset,
                                                const void* q_raster, const void* k_raster,
                                                const float* gamma_q, const float* gamma_k,
                                                float eps, float rope_theta, const void* dq_blk,
                                                const void* dk_blk, const void* dv_blk, void* dq,
                                                void* dk, void* dv, float* dgamma_q,
                                                float* dgamma_k, void* ws, size_t ws_bytes,
                                                bsa_stream_t stream);

/* ---- Sequence-parallel (Ulysses) form of the relayouts --------------------------------
 * Source: "LongCat-Video : Generate 1 minute long AI videos with this model", section
 * "How to run it" (multi-GPU inference with context parallelism, Ulysses) and the Meituan
 * talk, section 2.2 (the sparse attention is trained in parallel).  With the raster tensors of
 * a DiT split by frames over R ranks, rank r runs routing and attention for a slice of the
 * heads over the whole video: the sequence -> head exchange is folded into the prologue, which
 * reads every rank's frame shard directly (device pointers of peer GPUs, e.g. from
 * bsa_ipc_import), and the head -> sequence exchange into the inverse relayout, which writes
 * into every rank's shard.  No collective library call sits on this path; the caller orders
 * it with a barrier before the reads of peer shards and after the writes into them.
 *
 * Shard s of a raster tensor holds frames [s * shard_frames, (s + 1) * shard_frames) of the
 * grid being processed as bf16 [B, shard_frames * grid_h * grid_w, heads_total, D]; a call
 * processes raster heads head0 .. head0 + g->heads - 1 (the geometry describes the local
 * head slice).  Each shard pointer must be 16-byte aligned; a shard array holds n_shards
 * pointers (host memory, read during the call). */
#define BSA_MAX_SHARDS 8
typedef struct bsa_shards {
  int32_t n_shards;     /* 1 .. BSA_MAX_SHARDS; n_shards * shard_frames == frames */
  int32_t shard_frames; /* frames per shard */
  int32_t heads_total;  /* heads of each raster row */
  int32_t head0;        /* first raster head of this call */
} bsa_shards_t;

/* rope3d_qknorm_prologue reading its raster inputs from shards (q_shards / k_shards /
 * v_shards: arrays of n_shards pointers, or NULL to skip that tensor).  Outputs as there, for
 * the g->heads local heads. */
BSA_API bsa_status_t rope3d_qknorm_prologue_sharded(
    const bsa_geom_t* g, int32_t frames, int32_t t_offset, const bsa_shards_t* sh,
    const void* const* q_shards, const void* const* k_shards, const void* const* v_shards,
    const float* gamma_q, const float* gamma_k, float eps, float rope_theta, void* q_blk,
    void* k_blk, void* v_blk, float* q_pool, float* k_pool, bsa_stream_t stream);

/* rope3d_qknorm_prologue_bwd with sharded raster inputs (q_shards / k_shards, needed with a
 * gain) and outputs (dq_shards / dk_shards / dv_shards).  dgamma_q / dgamma_k are the
 * gradients over this call's heads only: the caller sums them over the ranks. */
BSA_API bsa_status_t rope3d_qknorm_prologue_bwd_sharded(
    const bsa_geom_t* g, int32_t frames, int32_t t_offset, const bsa_shards_t* sh,
    const void* const* q_shards, const void* const* k_shards, const float* gamma_q,
    const float* gamma_k, float eps, float rope_theta, const void* dq_blk, const void* dk_blk,
    const void* dv_blk, void* const* dq_shards, void* const* dk_shards, void* const* dv_shards,
    float* dgamma_q, float* dgamma_k, void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Inverse relayout of a blocked bf16 tensor (e.g. the attention output O) of the g->heads
 * local heads into raster shards (pad slots dropped): the head -> sequence exchange. */
BSA_API bsa_status_t bsa_blocked_to_raster_sharded(const bsa_geom_t* g, int32_t frames,
                                                   const bsa_shards_t* sh, const void* x_blk,
                                                   void* const* x_shards, bsa_stream_t stream);

/* CUDA IPC of device buffers between the processes of one node (plumbing for the shard
 * pointers above).  bsa_ipc_export writes BSA_IPC_HANDLE_BYTES bytes describing the device
 * allocation that holds dev_ptr and dev_ptr's offset in it; the exporting process must keep
 * the buffer alive until every importer has closed it.  bsa_ipc_import maps such a handle from
 * another process and returns the pointer to the same byte; bsa_ipc_close unmaps it.  A
 * process cannot import its own handle (BSA_ERR_CUDA). */
#define BSA_IPC_HANDLE_BYTES 128
BSA_API bsa_status_t bsa_ipc_export(const void* dev_ptr, void* handle);
BSA_API bsa_status_t bsa_ipc_import(const void* handle, void** dev_ptr);
BSA_API bsa_status_t bsa_ipc_close(void* dev_ptr);

/* Block-pooled top-r routing.
 * Sources: "LongCat-Video : Generate 1 minute long AI videos with this model", section
 * "Sparse attention" (blocks chosen by similarity); "LongCat-Video视频生成模型发布…",
 * section 块稀疏注意力（BSA） (keep the top-r key blocks).
 * For every (b, h, query block i): s_ij = qbar_i . kbar_j (fp32, unscaled) over all key
 * blocks j, -inf where the block-causal rule forbids j; keeps the top_r largest (ties to
 * the lower j), writes them ascending to idx with cnt = min(top_r, #allowed).
 * qbar/kbar are block means over valid tokens: taken from q_pool/k_pool when given
 * (e.g. from the prologue), else computed from q_blk/k_blk into the workspace.
 * kpool_cache: fp32 [B, H, NBc, D] means of the cached key blocks (required iff
 * cached_t > 0).  ws: BSA_WS_ROUTE bytes (may be NULL when both pools are given). */
BSA_API bsa_status_t bsa_route(const bsa_geom_t* g, int32_t top_r, const void* q_blk,
                       const void* k_blk, const float* q_pool, const float* k_pool,
                       const float* kpool_cache, int32_t* idx, int32_t* cnt, void* ws,
                       size_t ws_bytes, bsa_stream_t stream);

/* Routing variants for bsa_route_ex (bit flags).  The pages leave the routing rule open
 * ("LongCat-Video : Generate 1 minute long AI videos with this model", section "Sparse
 * attention", likens a block to one that always sits with its own table plus the meaningful
 * neighbouring ones); these are the variants of that reading.
 *   BSA_ROUTE_FORCE_SELF   every query block i keeps its own key block NBc + i; the other
 *                          top_r - 1 places go to the best of the rest (same tie rule).
 *   BSA_ROUTE_SHARED_HEADS key blocks ranked by s_ij = sum_h qbar_hi . kbar_hj; every head of
 *                          (b, i) gets that one selection (idx/cnt rows identical across h).
 *   BSA_ROUTE_POOL_SUM     block vectors are sums over the valid tokens (not means).
 *   BSA_ROUTE_POOL_MAX     block vectors are channel-wise maxima over the valid tokens.
 * A pooling flag pools q_blk / k_blk itself (q_pool / k_pool must be NULL, ws required);
 * kpool_cache must then hold the cached key blocks pooled the same way (bsa_block_pool). */
#define BSA_ROUTE_FORCE_SELF 1u
#define BSA_ROUTE_SHARED_HEADS 2u
#define BSA_ROUTE_POOL_SUM 4u
#define BSA_ROUTE_POOL_MAX 8u
/* bsa_route with variant flags (0 = bsa_route).  Unknown bits or both pooling flags:
 * BSA_ERR_INVALID_ARG. */
BSA_API bsa_status_t bsa_route_ex(const bsa_geom_t* g, int32_t top_r, uint32_t flags,
                                  const void* q_blk, const void* k_blk, const float* q_pool,
                                  const float* k_pool, const float* kpool_cache, int32_t* idx,
                                  int32_t* cnt, void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Block pooling of a blocked bf16 tensor x_blk [B, H, NB, BS, D] over `frames` frames
 * (NB = ceil(frames / blk_t) * NBh * NBw) into out fp32 [B, H, NB, D]: the mean
 * (BSA_POOL_MEAN), sum (BSA_POOL_SUM) or channel-wise maximum (BSA_POOL_MAX) over each
 * block's valid tokens (pad slots excluded).  Used to pool a cache for a pooling variant. */
#define BSA_POOL_MEAN 0
#define BSA_POOL_SUM 1
#define BSA_POOL_MAX 2
BSA_API bsa_status_t bsa_block_pool(const bsa_geom_t* g, int32_t frames, int32_t mode,
                                    const void* x_blk, float* out, bsa_stream_t stream);

/* Sparse attention forward over the selected blocks (tcgen05 tensor cores, TMA).
 * Source: "LongCat-Video视频生成模型发布…", section 块稀疏注意力（BSA）.
 * For every (b, h, query block i) and valid query slot:
 *   O = softmax(q K_S^T * scale) V_S, LSE = log sum exp(q K_S^T * scale), over the valid
 *   key tokens of the blocks S = idx[b,h,i,0:cnt].  Pad query slots get O = 0, LSE = -inf;
 *   cnt = 0 gives O = 0, LSE = -inf.
 * q_blk: blocked over the current frames; k_blk/v_blk: current key blocks; k_cache_blk /
 * v_cache_blk: blocked over cached_t frames (required iff cached_t > 0).  bf16 operands,
 * fp32 accumulation, O rounded to bf16.  All blocked tensors 16-byte aligned. */
BSA_API bsa_status_t bsa_attn_fwd(const bsa_geom_t* g, int32_t top_r, const void* q_blk,
                          const void* k_blk, const void* v_blk, const void* k_cache_blk,
                          const void* v_cache_blk, const int32_t* idx, const int32_t* cnt,
                          void* o_blk, float* lse, bsa_stream_t stream);

/* Sparse attention backward for a fixed routing (the forward's idx/cnt).
 * Source: "LongCat-Video 高效長視頻生成探索世界模型的第壹步", section 2.2 (forward and
 * backward of the sparse attention for training).  With P the softmax of the forward and
 * Delta = rowsum(dO * O):  dV_j += P^T dO,  dS = P * (dO V^T - Delta),
 * dQ_i += scale * dS K_j,  dK_j += scale * dS^T Q_i, summed over the selected pairs.
 * Gradients reach current keys/values only (cached ones are constants).  Outputs dq_blk,
 * dk_blk, dv_blk are bf16 blocked (pad slots 0); ws: BSA_WS_BWD bytes.
 * Block size: the backward takes 128-token blocks only (the forward also takes 32);
 * a geometry with BS = 32 returns BSA_ERR_UNSUPPORTED before any launch. */
BSA_API bsa_status_t bsa_attn_bwd(const bsa_geom_t* g, int32_t top_r, const void* q_blk,
                          const void* k_blk, const void* v_blk, const void* k_cache_blk,
                          const void* v_cache_blk, const void* o_blk, const float* lse,
                          const void* do_blk, const int32_t* idx, const int32_t* cnt,
                          void* dq_blk, void* dk_blk, void* dv_blk, void* ws,
                          size_t ws_bytes, bsa_stream_t stream);

/* Per-kernel timing for benchmarks (not part of the method; no page counterpart).
 * bsa_kernel_timing(1) starts it, (0) stops it; either call discards what was recorded.
 * While on, bsa_attn_fwd and bsa_attn_bwd record a CUDA event pair on their own stream
 * around each attention kernel they launch.  bsa_kernel_times(launches, total_ms) waits for
 * those events and fills BSA_NUM_TIMED entries (index BSA_TIMED_*): launches timed and their
 * summed milliseconds since the last call; the caller owns both arrays.  The library keeps
 * and reuses the events (host-side bookkeeping only; no device memory).  Off by default. */
#define BSA_TIMED_FWD 0
#define BSA_TIMED_BWD_DKDV 1
#define BSA_TIMED_BWD_DQ 2
#define BSA_NUM_TIMED 3
BSA_API bsa_status_t bsa_kernel_timing(int32_t on);
BSA_API bsa_status_t bsa_kernel_times(int32_t* launches, float* total_ms);
/* As bsa_kernel_times, plus the shortest and the median launch of each kernel (min_ms,
 * median_ms: BSA_NUM_TIMED entries each, or NULL); 0 for a kernel with no launch. */
BSA_API bsa_status_t bsa_kernel_time_stats(int32_t* launches, float* total_ms, float* min_ms,
                                           float* median_ms);

/* Waits for `stream`, then reads and clears the current device's status word.
 * Returns BSA_OK, BSA_ERR_TIMEOUT or BSA_ERR_BAD_INDEX (or BSA_ERR_CUDA). */
BSA_API bsa_status_t bsa_device_status(bsa_stream_t stream);

/* Routing without a caller workspace, for callers that cannot allocate device memory when they
 * route (a serving engine that reserved the whole device up front, a host framework whose
 * allocator owns all memory, a latency-critical path where cudaMalloc could synchronise the
 * device).  Same result as bsa_route with q_pool = k_pool = NULL (means computed from q_blk and
 * k_blk); the means live in a 16 MiB array inside the library, held on every device that loads
 * it until the process exits.  Rejects geometries with B*H*NBq*D*8 > 16 MiB (after 256-byte
 * rounding of each half) with BSA_ERR_UNSUPPORTED.  Allocates nothing.  The first call on a
 * device looks up that array's device address (cudaGetSymbolAddress) and caches it with the
 * current CUDA context: make it before any stream capture.  After cudaDeviceReset the next
 * call sees a new context and looks the address up again (make that call outside a capture
 * too).  Calls share the array, so calls that overlap on the GPU race.
 * No page counterpart: this entry point exists for callers that cannot allocate. */
BSA_API bsa_status_t bsa_route_noalloc(const bsa_geom_t* g, int32_t top_r, const void* q_blk,
                                       const void* k_blk, const float* kpool_cache, int32_t* idx,
                                       int32_t* cnt, bsa_stream_t stream);

/* Failure-path self test: enqueues one kernel that waits, through the same bounded wait every
 * kernel uses, on a barrier that nothing signals; after `limit_us` microseconds (1..1e6) it
 * gives up and records a timeout, which the next bsa_device_status() returns as
 * BSA_ERR_TIMEOUT.  The device stays usable.  No page counterpart: this tests the library's
 * own hang protection without hanging the GPU. */
BSA_API bsa_status_t bsa_selftest_bounded_wait(int32_t limit_us, bsa_stream_t stream);

/* Static string for a status code. */
BSA_API const char* bsa_error_string(bsa_status_t s);

/* Detail of the last argument error on the calling thread ("" if none). */
BSA_API const char* bsa_last_error_detail(void);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H_ */
