// bsa_lib.cu -- libbsa.so: the C ABI declared in include/bsa.h.
//
// One translation unit (the kernel files are included below) so that every kernel shares
// the single per-device status word without relocatable device code.  Host code here
// validates arguments, derives the block geometry, encodes TMA tensor maps and enqueues the
// kernels on the caller's stream.  It allocates no device memory.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "common.cuh"
#include "timing.cuh"

#include "prologue.cu"
#include "route.cu"
#include "attn_fwd.cu"
#include "attn_bwd.cu"
#include "cache_append.cu"

namespace bsa {

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing ever arrives on,
// with the caller's limit, through the same mbar_wait every kernel uses; it must give up,
// record DEV_TIMEOUT and return (the context stays usable).
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  mbar_wait(&bar, 0, &abort_flag, limit_ns);
}

namespace {

thread_local std::string t_detail;

bsa_status_t fail(bsa_status_t s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_detail = buf;
  return s;
}

bsa_status_t cuda_fail(cudaError_t e, const char* where) {
  return fail(BSA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- device checks (cached)
struct DevInfo {
  int checked = 0;  // 0 unknown, 1 ok, -1 unsupported
  int n_sm = 0;
};
DevInfo g_dev[64];
std::mutex g_dev_mu;

bsa_status_t check_device(int* n_sm) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(BSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (d.checked == 0) {
    int major = 0, minor = 0, sms = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.checked = (major == 10 && minor == 0) ? 1 : -1;
    d.n_sm = sms;
  }
  if (d.checked < 0)
    return fail(BSA_ERR_UNSUPPORTED, "libbsa is built for sm_100a only (B200)");
  if (n_sm) *n_sm = d.n_sm;
  return BSA_OK;
}

// ---------------------------------------------------------------- geometry
bsa_status_t make_geo(const bsa_geom_t* gi, Geo* out) {
  if (gi == nullptr) return fail(BSA_ERR_INVALID_ARG, "geometry is NULL");
  const bsa_geom_t& a = *gi;
  if (a.batch < 1 || a.heads < 1 || a.t_frames < 1 || a.grid_h < 1 || a.grid_w < 1)
    return fail(BSA_ERR_INVALID_ARG, "batch, heads, t_frames, grid_h, grid_w must be >= 1");
  if (a.head_dim != 64 && a.head_dim != 128)
    return fail(BSA_ERR_UNSUPPORTED, "head_dim %d (supported: 64, 128)", a.head_dim);
  if (a.blk_t < 1 || a.blk_h < 1 || a.blk_w < 1)
    return fail(BSA_ERR_INVALID_ARG, "block dims must be >= 1");
  const long bs = (long)a.blk_t * a.blk_h * a.blk_w;
  if (bs != 32 && bs != 128)
    return fail(BSA_ERR_UNSUPPORTED, "block size %ld tokens (supported: 32, 128)", bs);
  if (a.cached_t < 0 || a.cached_t % a.blk_t)
    return fail(BSA_ERR_INVALID_ARG, "cached_t %d must be >= 0 and a multiple of blk_t",
                a.cached_t);
  if (a.causal_chunk_t < 0 || (a.causal_chunk_t && a.causal_chunk_t % a.blk_t))
    return fail(BSA_ERR_INVALID_ARG, "causal_chunk_t %d must be 0 or a multiple of blk_t",
                a.causal_chunk_t);
  if (a.cond_t < 0 || a.cond_t % a.blk_t)
    return fail(BSA_ERR_INVALID_ARG, "cond_t %d must be >= 0 and a multiple of blk_t", a.cond_t);
  if (!(a.softmax_scale >= 0.f) || std::isinf(a.softmax_scale))
    return fail(BSA_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  Geo g;
  g.B = a.batch; g.H = a.heads; g.D = a.head_dim;
  g.T = a.t_frames; g.GH = a.grid_h; g.GW = a.grid_w; g.Tc = a.cached_t;
  g.bt = a.blk_t; g.bh = a.blk_h; g.bw = a.blk_w; g.BS = (int)bs;
  g.lbh = 0;
  while ((1 << g.lbh) < g.bh) ++g.lbh;
  g.lbw = 0;
  while ((1 << g.lbw) < g.bw) ++g.lbw;
  g.nbh = (a.grid_h + a.blk_h - 1) / a.blk_h;
  g.nbw = (a.grid_w + a.blk_w - 1) / a.blk_w;
  g.nbt_q = (a.t_frames + a.blk_t - 1) / a.blk_t;
  g.nbt_c = a.cached_t / a.blk_t;
  const long per_t = (long)g.nbh * g.nbw;
  const long nbq = per_t * g.nbt_q, nbc = per_t * g.nbt_c;
  if (nbq + nbc > 4096)
    return fail(BSA_ERR_UNSUPPORTED, "%ld key blocks per head (supported: <= 4096)", nbq + nbc);
  const long rows = (long)g.B * g.H * (nbq + nbc) * bs;
  if (rows >= (1L << 31) - 256)
    return fail(BSA_ERR_UNSUPPORTED, "problem too large for 32-bit TMA row coordinates");
  g.NBq = (int)nbq; g.NBc = (int)nbc; g.NBk = (int)(nbq + nbc);
  g.chunk = a.causal_chunk_t;
  g.cond = a.cond_t;
  g.scale = a.softmax_scale > 0.f ? a.softmax_scale : 1.0f / std::sqrt((float)a.head_dim);
  *out = g;
  return BSA_OK;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ---------------------------------------------------------------- TMA tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

bsa_status_t get_encoder(EncodeTiledFn* fn) {
  std::call_once(g_encode_once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(f);
  });
  if (!g_encode) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  *fn = g_encode;
  return BSA_OK;
}

// 2D view [rows, D] of a blocked bf16 tensor, box = [64 columns, box_rows rows], 128B swizzle.
bsa_status_t encode_blocked(CUtensorMap* map, const void* ptr, long rows, int D, int box_rows) {
  EncodeTiledFn enc;
  bsa_status_t st = get_encoder(&enc);
  if (st != BSA_OK) return st;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return BSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct RouteWs {
  size_t qpool, kpool, total;
};
RouteWs route_ws(const Geo& g) {
  RouteWs w;
  w.qpool = 0;
  w.kpool = align256((size_t)g.B * g.H * g.NBq * g.D * sizeof(float));
  w.total = w.kpool + align256((size_t)g.B * g.H * g.NBq * g.D * sizeof(float));
  return w;
}

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" {

int32_t bsa_abi_version(void) { return BSA_ABI_VERSION; }

const char* bsa_error_string(bsa_status_t s) {
  switch (s) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported device or shape";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
    case BSA_ERR_BAD_INDEX: return "block index or count out of range";
    case BSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

const char* bsa_last_error_detail(void) { return t_detail.c_str(); }

size_t bsa_workspace_size(const bsa_geom_t* gi, int32_t top_r, int32_t which) {
  Geo g;
  if (make_geo(gi, &g) != BSA_OK || top_r < 1) return 0;
  if (which == BSA_WS_ROUTE) return route_ws(g).total;
  if (which == BSA_WS_FWD) return 0;
  if (which == BSA_WS_BWD) return bwd_ws_layout(g, top_r).total;
  if (which == BSA_WS_PROLOGUE_BWD)
    return 2 * align256((size_t)prologue_bwd_ctas(g, (g.T + g.bt - 1) / g.bt) * g.D * sizeof(float));
  return 0;
}

bsa_status_t rope3d_qknorm_prologue(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                    const void* q_raster, const void* k_raster,
                                    const void* v_raster, const float* gamma_q,
                                    const float* gamma_k, float eps, float rope_theta,
                                    void* q_blk, void* k_blk, void* v_blk, float* q_pool,
                                    float* k_pool, bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (frames < 1) return fail(BSA_ERR_INVALID_ARG, "frames must be >= 1");
  if (t_offset < 0) return fail(BSA_ERR_INVALID_ARG, "t_offset must be >= 0");
  if (!(eps >= 0.f) || !(rope_theta >= 0.f) || std::isinf(rope_theta))
    return fail(BSA_ERR_INVALID_ARG, "eps and rope_theta must be finite and >= 0");
  const void* xs[3] = {q_raster, k_raster, v_raster};
  void* ys[3] = {q_blk, k_blk, v_blk};
  bool any = false;
  for (int i = 0; i < 3; ++i) {
    if ((xs[i] == nullptr) != (ys[i] == nullptr))
      return fail(BSA_ERR_INVALID_ARG, "input %d and its output must both be given or both NULL", i);
    if (xs[i] && (!aligned(xs[i], 16) || !aligned(ys[i], 16)))
      return fail(BSA_ERR_INVALID_ARG, "tensor %d not 16-byte aligned", i);
    any |= xs[i] != nullptr;
  }
  if (!any) return fail(BSA_ERR_INVALID_ARG, "no tensor to process");
  if ((q_pool && !q_raster) || (k_pool && !k_raster))
    return fail(BSA_ERR_INVALID_ARG, "a pool output needs its tensor");
  if ((q_pool && !aligned(q_pool, 16)) || (k_pool && !aligned(k_pool, 16)))
    return fail(BSA_ERR_INVALID_ARG, "pool outputs must be 16-byte aligned");
  if (((long)frames * g.GH * g.GW) * (long)g.B * g.H * g.D >= (1L << 40))
    return fail(BSA_ERR_UNSUPPORTED, "tensor too large");
  st = check_device(nullptr);
  if (st != BSA_OK) return st;
  PrologueArgs a;
  a.g = g;
  a.frames = frames;
  a.t_offset = t_offset;
  a.nbt = (frames + g.bt - 1) / g.bt;
  for (int i = 0; i < 3; ++i) {
    a.x[i] = static_cast<const __nv_bfloat16*>(xs[i]);
    a.y[i] = static_cast<__nv_bfloat16*>(ys[i]);
  }
  a.gamma[0] = gamma_q;
  a.gamma[1] = gamma_k;
  a.pool[0] = q_pool;
  a.pool[1] = k_pool;
  a.eps = eps;
  a.theta = rope_theta;
  a.dh = 2 * (g.D / 6);
  a.dw = a.dh;
  a.dt = g.D - 2 * a.dh;
  cudaError_t e = launch_prologue(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
  return BSA_OK;
}

bsa_status_t rope3d_qknorm_prologue_bwd(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                        const void* q_raster, const void* k_raster,
                                        const float* gamma_q, const float* gamma_k, float eps,
                                        float rope_theta, const void* dq_blk, const void* dk_blk,
                                        const void* dv_blk, void* dq, void* dk, void* dv,
                                        float* dgamma_q, float* dgamma_k, void* ws, size_t ws_bytes,
                                        bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (frames < 1) return fail(BSA_ERR_INVALID_ARG, "frames must be >= 1");
  if (t_offset < 0) return fail(BSA_ERR_INVALID_ARG, "t_offset must be >= 0");
  if (!(eps >= 0.f) || !(rope_theta >= 0.f) || std::isinf(rope_theta))
    return fail(BSA_ERR_INVALID_ARG, "eps and rope_theta must be finite and >= 0");
  const void* dz[3] = {dq_blk, dk_blk, dv_blk};
  void* dxs[3] = {dq, dk, dv};
  const void* xs[2] = {q_raster, k_raster};
  const float* gams[2] = {gamma_q, gamma_k};
  float* dgs[2] = {dgamma_q, dgamma_k};
  bool any = false, any_gain = false;
  for (int i = 0; i < 3; ++i) {
    if ((dz[i] == nullptr) != (dxs[i] == nullptr))
      return fail(BSA_ERR_INVALID_ARG, "gradient %d and its output must both be given or both NULL", i);
    if (dz[i] && (!aligned(dz[i], 16) || !aligned(dxs[i], 16)))
      return fail(BSA_ERR_INVALID_ARG, "tensor %d not 16-byte aligned", i);
    any |= dz[i] != nullptr;
  }
  if (!any) return fail(BSA_ERR_INVALID_ARG, "no tensor to process");
  for (int i = 0; i < 2; ++i) {
    if (dz[i] && gams[i]) {
      if (!xs[i] || !dgs[i])
        return fail(BSA_ERR_INVALID_ARG, "with a gain, tensor %d needs its raster input and a dgamma output", i);
      if (!aligned(xs[i], 16)) return fail(BSA_ERR_INVALID_ARG, "raster input %d not 16-byte aligned", i);
      any_gain = true;
    }
  }
  if (((long)frames * g.GH * g.GW) * (long)g.B * g.H * g.D >= (1L << 40))
    return fail(BSA_ERR_UNSUPPORTED, "tensor too large");
  const int nbt = (frames + g.bt - 1) / g.bt;
  const size_t part_bytes = align256((size_t)prologue_bwd_ctas(g, nbt) * g.D * sizeof(float));
  if (any_gain && (ws == nullptr || ws_bytes < 2 * part_bytes || !aligned(ws, 256)))
    return fail(BSA_ERR_WORKSPACE, "prologue backward needs %zu workspace bytes (256-byte aligned)",
                2 * part_bytes);
  st = check_device(nullptr);
  if (st != BSA_OK) return st;
  PrologueBwdArgs a;
  PrologueArgs& f = a.f;
  f.g = g;
  f.frames = frames;
  f.t_offset = t_offset;
  f.nbt = nbt;
  for (int i = 0; i < 3; ++i) { f.x[i] = nullptr; f.y[i] = nullptr; }
  f.gamma[0] = dq_blk ? gamma_q : nullptr;
  f.gamma[1] = dk_blk ? gamma_k : nullptr;
  f.pool[0] = f.pool[1] = nullptr;
  f.eps = eps;
  f.theta = rope_theta;
  f.dh = 2 * (g.D / 6);
  f.dw = f.dh;
  f.dt = g.D - 2 * f.dh;
  for (int i = 0; i < 3; ++i) {
    a.dz[i] = static_cast<const __nv_bfloat16*>(dz[i]);
    a.dx[i] = static_cast<__nv_bfloat16*>(dxs[i]);
  }
  for (int i = 0; i < 2; ++i) {
    a.x[i] = static_cast<const __nv_bfloat16*>(xs[i]);
    a.part[i] = (dz[i] && gams[i]) ? reinterpret_cast<float*>(static_cast<char*>(ws) + i * part_bytes)
                                   : nullptr;
    if (!(dz[i] && gams[i])) dgs[i] = nullptr;
  }
  cudaError_t e = launch_prologue_bwd(a, dgs, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prologue backward launch");
  return BSA_OK;
}

bsa_status_t bsa_cache_append(const bsa_geom_t* gi, const void* kc_blk, const void* vc_blk,
                              const float* kc_pool, const void* k_blk, const void* v_blk,
                              const float* k_pool, void* kc_new, void* vc_new, float* kc_pool_new,
                              bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (g.T % g.bt)
    return fail(BSA_ERR_UNSUPPORTED, "t_frames %d must be a multiple of blk_t to extend a cache", g.T);
  if (!k_blk || !v_blk || !kc_new || !vc_new)
    return fail(BSA_ERR_INVALID_ARG, "k_blk, v_blk, kc_new and vc_new are required");
  if (g.NBc > 0 && (!kc_blk || !vc_blk))
    return fail(BSA_ERR_INVALID_ARG, "kc_blk and vc_blk are required when cached_t > 0");
  if ((kc_pool_new != nullptr) != (k_pool != nullptr) || (kc_pool_new && g.NBc > 0 && !kc_pool))
    return fail(BSA_ERR_INVALID_ARG, "block means: give k_pool and kc_pool_new (and kc_pool when cached_t > 0) or none");
  const void* ptrs[9] = {kc_blk, vc_blk, kc_pool, k_blk, v_blk, k_pool, kc_new, vc_new, kc_pool_new};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int n_sm = 0;
  st = check_device(&n_sm);
  if (st != BSA_OK) return st;
  const int bh = g.B * g.H;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t tile = (size_t)g.BS * g.D * 2;
  cudaError_t e = launch_cache_append(kc_blk, k_blk, kc_new, bh, g.NBc, g.NBq, tile, n_sm, s);
  if (e == cudaSuccess) e = launch_cache_append(vc_blk, v_blk, vc_new, bh, g.NBc, g.NBq, tile, n_sm, s);
  if (e == cudaSuccess && kc_pool_new)
    e = launch_cache_append(kc_pool, k_pool, kc_pool_new, bh, g.NBc, g.NBq, (size_t)g.D * 4, n_sm, s);
  if (e != cudaSuccess) return cuda_fail(e, "cache append launch");
  return BSA_OK;
}

bsa_status_t bsa_route(const bsa_geom_t* gi, int32_t top_r, const void* q_blk,
                       const void* k_blk, const float* q_pool, const float* k_pool,
                       const float* kpool_cache, int32_t* idx, int32_t* cnt, void* ws,
                       size_t ws_bytes, bsa_stream_t stream) {
  return bsa_route_ex(gi, top_r, 0u, q_blk, k_blk, q_pool, k_pool, kpool_cache, idx, cnt, ws,
                      ws_bytes, stream);
}

bsa_status_t bsa_route_ex(const bsa_geom_t* gi, int32_t top_r, uint32_t flags, const void* q_blk,
                          const void* k_blk, const float* q_pool, const float* k_pool,
                          const float* kpool_cache, int32_t* idx, int32_t* cnt, void* ws,
                          size_t ws_bytes, bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (top_r < 1) return fail(BSA_ERR_INVALID_ARG, "top_r must be >= 1");
  const uint32_t known = BSA_ROUTE_FORCE_SELF | BSA_ROUTE_SHARED_HEADS | BSA_ROUTE_POOL_SUM |
                         BSA_ROUTE_POOL_MAX;
  if (flags & ~known) return fail(BSA_ERR_INVALID_ARG, "unknown route flags 0x%x", flags & ~known);
  const bool pool_sum = flags & BSA_ROUTE_POOL_SUM, pool_max = flags & BSA_ROUTE_POOL_MAX;
  if (pool_sum && pool_max) return fail(BSA_ERR_INVALID_ARG, "choose one pooling mode");
  const int pool_mode = pool_sum ? kPoolSum : pool_max ? kPoolMax : kPoolMean;
  if (pool_mode != kPoolMean && (q_pool || k_pool))
    return fail(BSA_ERR_INVALID_ARG, "a pooling flag pools q_blk / k_blk here: pass no q_pool / k_pool");
  if (!idx || !cnt) return fail(BSA_ERR_INVALID_ARG, "idx and cnt are required");
  if ((!q_pool && !q_blk) || (!k_pool && !k_blk))
    return fail(BSA_ERR_INVALID_ARG, "need q_blk or q_pool, and k_blk or k_pool");
  if (g.NBc > 0 && !kpool_cache)
    return fail(BSA_ERR_INVALID_ARG, "kpool_cache is required when cached_t > 0");
  const void* ptrs[5] = {q_blk, k_blk, q_pool, k_pool, kpool_cache};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(BSA_ERR_INVALID_ARG, "inputs must be 16-byte aligned");
  const RouteWs w = route_ws(g);
  if ((!q_pool || !k_pool) && (ws == nullptr || ws_bytes < w.total || !aligned(ws, 256)))
    return fail(BSA_ERR_WORKSPACE, "route needs %zu workspace bytes (256-byte aligned)", w.total);
  // one CTA covers all heads of its query rows when they share a selection: fewer rows per
  // CTA keep more SMs busy
  const int qt = (flags & BSA_ROUTE_SHARED_HEADS) ? std::min(select_rows_per_cta(g), 8)
                                                  : select_rows_per_cta(g);
  if (qt == 0) return fail(BSA_ERR_UNSUPPORTED, "%d key blocks do not fit the select kernel", g.NBk);
  int n_sm = 0;
  st = check_device(&n_sm);
  if (st != BSA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (!q_pool) {
    float* out = reinterpret_cast<float*>(static_cast<char*>(ws) + w.qpool);
    if ((e = launch_pool(static_cast<const __nv_bfloat16*>(q_blk), g.T, g.NBq, g, out, s, pool_mode)) != cudaSuccess)
      return cuda_fail(e, "pool launch");
    q_pool = out;
  }
  if (!k_pool) {
    float* out = reinterpret_cast<float*>(static_cast<char*>(ws) + w.kpool);
    if ((e = launch_pool(static_cast<const __nv_bfloat16*>(k_blk), g.T, g.NBq, g, out, s, pool_mode)) != cudaSuccess)
      return cuda_fail(e, "pool launch");
    k_pool = out;
  }
  SelectArgs a;
  a.g = g;
  a.r = top_r;
  a.flags = (flags & BSA_ROUTE_FORCE_SELF ? kRouteForceSelf : 0u) |
            (flags & BSA_ROUTE_SHARED_HEADS ? kRouteSharedHeads : 0u);
  a.qt = qt;
  a.qpool = q_pool;
  a.kpool = k_pool;
  a.kpool_cache = kpool_cache;
  a.idx = idx;
  a.cnt = cnt;
  if ((e = launch_select(a, s)) != cudaSuccess) return cuda_fail(e, "select launch");
  return BSA_OK;
}

bsa_status_t bsa_block_pool(const bsa_geom_t* gi, int32_t frames, int32_t mode,
                            const void* x_blk, float* out, bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (frames < 1) return fail(BSA_ERR_INVALID_ARG, "frames must be >= 1");
  if (mode != BSA_POOL_MEAN && mode != BSA_POOL_SUM && mode != BSA_POOL_MAX)
    return fail(BSA_ERR_INVALID_ARG, "unknown pooling mode %d", mode);
  if (!x_blk || !out) return fail(BSA_ERR_INVALID_ARG, "x_blk and out are required");
  if (!aligned(x_blk, 16) || !aligned(out, 16))
    return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int n_sm = 0;
  st = check_device(&n_sm);
  if (st != BSA_OK) return st;
  const int nb = ((frames + g.bt - 1) / g.bt) * g.nbh * g.nbw;
  const int m = mode == BSA_POOL_SUM ? kPoolSum : mode == BSA_POOL_MAX ? kPoolMax : kPoolMean;
  cudaError_t e = launch_pool(static_cast<const __nv_bfloat16*>(x_blk), frames, nb, g, out,
                              reinterpret_cast<cudaStream_t>(stream), m);
  if (e != cudaSuccess) return cuda_fail(e, "pool launch");
  return BSA_OK;
}

bsa_status_t bsa_attn_fwd(const bsa_geom_t* gi, int32_t top_r, const void* q_blk,
                          const void* k_blk, const void* v_blk, const void* k_cache_blk,
                          const void* v_cache_blk, const int32_t* idx, const int32_t* cnt,
                          void* o_blk, float* lse, bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (top_r < 1) return fail(BSA_ERR_INVALID_ARG, "top_r must be >= 1");
  if (!q_blk || !k_blk || !v_blk || !idx || !cnt || !o_blk || !lse)
    return fail(BSA_ERR_INVALID_ARG, "q, k, v, idx, cnt, o and lse are required");
  if (g.NBc > 0 && (!k_cache_blk || !v_cache_blk))
    return fail(BSA_ERR_INVALID_ARG, "k_cache_blk and v_cache_blk are required when cached_t > 0");
  const void* ptrs[7] = {q_blk, k_blk, v_blk, k_cache_blk, v_cache_blk, o_blk, lse};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  int n_sm = 0;
  st = check_device(&n_sm);
  if (st != BSA_OK) return st;
  const long bh = (long)g.B * g.H;
  CUtensorMap maps[5];
  if ((st = encode_blocked(&maps[0], q_blk, bh * g.NBq * g.BS, g.D, kTileM)) != BSA_OK) return st;
  if ((st = encode_blocked(&maps[1], k_blk, bh * g.NBq * g.BS, g.D, g.BS)) != BSA_OK) return st;
  if ((st = encode_blocked(&maps[2], v_blk, bh * g.NBq * g.BS, g.D, g.BS)) != BSA_OK) return st;
  if (g.NBc > 0) {
    if ((st = encode_blocked(&maps[3], k_cache_blk, bh * g.NBc * g.BS, g.D, g.BS)) != BSA_OK) return st;
    if ((st = encode_blocked(&maps[4], v_cache_blk, bh * g.NBc * g.BS, g.D, g.BS)) != BSA_OK) return st;
  } else {
    maps[3] = maps[1];
    maps[4] = maps[2];
  }
  FwdParams p;
  p.g = g;
  p.r = top_r;
  p.n_items = (int)(bh * g.NBq);
  p.idx = idx;
  p.cnt = cnt;
  p.o = static_cast<__nv_bfloat16*>(o_blk);
  p.lse = lse;
  cudaEvent_t t0;
  const int tw = timed_begin(BSA_TIMED_FWD, reinterpret_cast<cudaStream_t>(stream), &t0);
  cudaError_t e = launch_fwd(maps, p, n_sm, reinterpret_cast<cudaStream_t>(stream));
  timed_end(tw, reinterpret_cast<cudaStream_t>(stream), t0);
  if (e != cudaSuccess) return cuda_fail(e, "fwd launch");
  return BSA_OK;
}

bsa_status_t bsa_attn_bwd(const bsa_geom_t* gi, int32_t top_r, const void* q_blk,
                          const void* k_blk, const void* v_blk, const void* k_cache_blk,
                          const void* v_cache_blk, const void* o_blk, const float* lse,
                          const void* do_blk, const int32_t* idx, const int32_t* cnt,
                          void* dq_blk, void* dk_blk, void* dv_blk, void* ws, size_t ws_bytes,
                          bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (top_r < 1) return fail(BSA_ERR_INVALID_ARG, "top_r must be >= 1");
  if (!q_blk || !k_blk || !v_blk || !o_blk || !lse || !do_blk || !idx || !cnt || !dq_blk ||
      !dk_blk || !dv_blk)
    return fail(BSA_ERR_INVALID_ARG, "missing tensor argument");
  if (g.NBc > 0 && (!k_cache_blk || !v_cache_blk))
    return fail(BSA_ERR_INVALID_ARG, "k_cache_blk and v_cache_blk are required when cached_t > 0");
  const void* ptrs[11] = {q_blk, k_blk, v_blk, k_cache_blk, v_cache_blk, o_blk, lse, do_blk,
                          dq_blk, dk_blk, dv_blk};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(BSA_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
  const BwdWs w = bwd_ws_layout(g, top_r);
  if (ws == nullptr || ws_bytes < w.total || !aligned(ws, 256))
    return fail(BSA_ERR_WORKSPACE, "bwd needs %zu workspace bytes (256-byte aligned)", w.total);
  int n_sm = 0;
  st = check_device(&n_sm);
  if (st != BSA_OK) return st;
  if (g.BS != 128)
    return fail(BSA_ERR_UNSUPPORTED, "backward supports 128-token blocks (got %d)", g.BS);
  const long bh = (long)g.B * g.H;
  CUtensorMap maps[6];
  if ((st = encode_blocked(&maps[0], q_blk, bh * g.NBq * g.BS, g.D, kTileM)) != BSA_OK) return st;
  if ((st = encode_blocked(&maps[1], k_blk, bh * g.NBq * g.BS, g.D, g.BS)) != BSA_OK) return st;
  if ((st = encode_blocked(&maps[2], v_blk, bh * g.NBq * g.BS, g.D, g.BS)) != BSA_OK) return st;
  if (g.NBc > 0) {
    if ((st = encode_blocked(&maps[3], k_cache_blk, bh * g.NBc * g.BS, g.D, g.BS)) != BSA_OK) return st;
    if ((st = encode_blocked(&maps[4], v_cache_blk, bh * g.NBc * g.BS, g.D, g.BS)) != BSA_OK) return st;
  } else {
    maps[3] = maps[1];
    maps[4] = maps[2];
  }
  if ((st = encode_blocked(&maps[5], do_blk, bh * g.NBq * g.BS, g.D, kTileM)) != BSA_OK) return st;
  BwdPtrs P;
  P.q = q_blk; P.k = k_blk; P.v = v_blk; P.kc = k_cache_blk; P.vc = v_cache_blk;
  P.o = o_blk; P.lse = lse; P.dO = do_blk; P.idx = idx; P.cnt = cnt;
  P.dq = dq_blk; P.dk = dk_blk; P.dv = dv_blk; P.ws = static_cast<char*>(ws);
  st = run_bwd(g, top_r, P, w, maps, n_sm, reinterpret_cast<cudaStream_t>(stream));
  if (st != BSA_OK) return fail(st, "bwd launch failed");
  return BSA_OK;
}

bsa_status_t bsa_selftest_bounded_wait(int32_t limit_us, bsa_stream_t stream) {
  t_detail.clear();
  if (limit_us < 1 || limit_us > 1000000)
    return fail(BSA_ERR_INVALID_ARG, "limit_us must be in [1, 1e6]");
  bsa_status_t st = check_device(nullptr);
  if (st != BSA_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_us * 1000ull);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return BSA_OK;
}

bsa_status_t bsa_kernel_timing(int32_t on) {
  t_detail.clear();
  KernelTimer& t = kernel_timer();
  std::lock_guard<std::mutex> lk(t.mu);
  for (auto& v : t.pending) {  // drop what was recorded before (events go back to the pool)
    for (auto& pr : v) {
      cudaEventSynchronize(pr.second);
      t.pool.push_back(pr.first);
      t.pool.push_back(pr.second);
    }
    v.clear();
  }
  t.on.store(on ? 1 : 0);
  return BSA_OK;
}

bsa_status_t bsa_kernel_times(int32_t* launches, float* total_ms) {
  t_detail.clear();
  if (!launches || !total_ms) return fail(BSA_ERR_INVALID_ARG, "launches and total_ms are required");
  KernelTimer& t = kernel_timer();
  std::lock_guard<std::mutex> lk(t.mu);
  bsa_status_t st = BSA_OK;
  for (int k = 0; k < kNumTimed; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.f;
    for (auto& pr : t.pending[k]) {
      float ms = 0.f;
      cudaError_t e = cudaEventSynchronize(pr.second);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
      if (e != cudaSuccess && st == BSA_OK) st = cuda_fail(e, "kernel timing event");
      ++launches[k];
      total_ms[k] += ms;
      t.pool.push_back(pr.first);
      t.pool.push_back(pr.second);
    }
    t.pending[k].clear();
  }
  return st;
}

bsa_status_t bsa_device_status(bsa_stream_t stream) {
  t_detail.clear();
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&v, g_dev_status, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read status word");
  if (v) {
    e = cudaMemcpyToSymbol(g_dev_status, &zero, sizeof(zero));
    if (e != cudaSuccess) return cuda_fail(e, "clear status word");
  }
  if (v & DEV_TIMEOUT) return fail(BSA_ERR_TIMEOUT, "device status 0x%x", v);
  if (v & DEV_BAD_INDEX) return fail(BSA_ERR_BAD_INDEX, "device status 0x%x", v);
  return BSA_OK;
}

}  // extern "C"

#include "route_noalloc.cu"
