// bsa_lib.cu -- libbsa.so: the C ABI declared in include/bsa.h.
//
// One translation unit (the kernel files are included below) so that every kernel shares
// the single per-device status word without relocatable device code.  Host code here
// validates arguments, derives the block geometry, encodes TMA tensor maps and enqueues the
// kernels on the caller's stream.  It allocates no device memory.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

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

// Shards of the raster tensors: NULL = one shard holding every frame and head of the call.
static bsa_status_t make_shards(const Geo& g, int32_t frames, const bsa_shards_t* sd,
                                RasterShards* out) {
  RasterShards r{1, frames, g.H, 0};
  if (sd) {
    if (sd->n_shards < 1 || sd->n_shards > kMaxShards)
      return fail(BSA_ERR_INVALID_ARG, "n_shards %d (supported: 1..%d)", sd->n_shards, kMaxShards);
    if (sd->shard_frames < 1 || (long)sd->n_shards * sd->shard_frames != frames)
      return fail(BSA_ERR_INVALID_ARG, "n_shards * shard_frames must equal frames (%d)", frames);
    if (sd->head0 < 0 || sd->heads_total < 1 || (long)sd->head0 + g.H > sd->heads_total)
      return fail(BSA_ERR_INVALID_ARG, "heads head0 .. head0 + heads - 1 must lie in 0 .. heads_total - 1");
    r = RasterShards{sd->n_shards, sd->shard_frames, sd->heads_total, sd->head0};
  }
  if (((long)r.frames * g.GH * g.GW) * (long)g.B * r.h_stride * g.D >= (1L << 40))
    return fail(BSA_ERR_UNSUPPORTED, "tensor too large");
  *out = r;
  return BSA_OK;
}

// Every shard pointer of a given tensor present and 16-byte aligned.
static bool shard_ptrs_ok(const void* const* p, int n) {
  for (int s = 0; s < n; ++s)
    if (p[s] == nullptr || !aligned(p[s], 16)) return false;
  return true;
}

static bsa_status_t prologue_impl(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                  const bsa_shards_t* sd, const void* const* const xsh[3],
                                  const float* gamma_q, const float* gamma_k, float eps,
                                  float rope_theta, void* q_blk, void* k_blk, void* v_blk,
                                  float* q_pool, float* k_pool, bsa_stream_t stream) {
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (frames < 1) return fail(BSA_ERR_INVALID_ARG, "frames must be >= 1");
  if (t_offset < 0) return fail(BSA_ERR_INVALID_ARG, "t_offset must be >= 0");
  if (!(eps >= 0.f) || !(rope_theta >= 0.f) || std::isinf(rope_theta))
    return fail(BSA_ERR_INVALID_ARG, "eps and rope_theta must be finite and >= 0");
  RasterShards sh;
  if ((st = make_shards(g, frames, sd, &sh)) != BSA_OK) return st;
  void* ys[3] = {q_blk, k_blk, v_blk};
  bool any = false;
  for (int i = 0; i < 3; ++i) {
    if ((xsh[i] == nullptr) != (ys[i] == nullptr))
      return fail(BSA_ERR_INVALID_ARG, "input %d and its output must both be given or both NULL", i);
    if (xsh[i] && (!shard_ptrs_ok(xsh[i], sh.n) || !aligned(ys[i], 16)))
      return fail(BSA_ERR_INVALID_ARG, "tensor %d: a shard is NULL or a tensor is not 16-byte aligned", i);
    any |= xsh[i] != nullptr;
  }
  if (!any) return fail(BSA_ERR_INVALID_ARG, "no tensor to process");
  if ((q_pool && !xsh[0]) || (k_pool && !xsh[1]))
    return fail(BSA_ERR_INVALID_ARG, "a pool output needs its tensor");
  if ((q_pool && !aligned(q_pool, 16)) || (k_pool && !aligned(k_pool, 16)))
    return fail(BSA_ERR_INVALID_ARG, "pool outputs must be 16-byte aligned");
  st = check_device(nullptr);
  if (st != BSA_OK) return st;
  PrologueArgs a;
  a.g = g;
  a.frames = frames;
  a.t_offset = t_offset;
  a.nbt = (frames + g.bt - 1) / g.bt;
  a.sh = sh;
  for (int i = 0; i < 3; ++i) {
    for (int s2 = 0; s2 < kMaxShards; ++s2)
      a.x[i][s2] = (xsh[i] && s2 < sh.n) ? static_cast<const __nv_bfloat16*>(xsh[i][s2]) : nullptr;
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

bsa_status_t rope3d_qknorm_prologue(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                    const void* q_raster, const void* k_raster,
                                    const void* v_raster, const float* gamma_q,
                                    const float* gamma_k, float eps, float rope_theta,
                                    void* q_blk, void* k_blk, void* v_blk, float* q_pool,
                                    float* k_pool, bsa_stream_t stream) {
  const void* one[3][1] = {{q_raster}, {k_raster}, {v_raster}};
  const void* const* xsh[3] = {q_raster ? one[0] : nullptr, k_raster ? one[1] : nullptr,
                               v_raster ? one[2] : nullptr};
  return prologue_impl(gi, frames, t_offset, nullptr, xsh, gamma_q, gamma_k, eps, rope_theta,
                       q_blk, k_blk, v_blk, q_pool, k_pool, stream);
}

bsa_status_t rope3d_qknorm_prologue_sharded(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                            const bsa_shards_t* sh, const void* const* q_shards,
                                            const void* const* k_shards,
                                            const void* const* v_shards, const float* gamma_q,
                                            const float* gamma_k, float eps, float rope_theta,
                                            void* q_blk, void* k_blk, void* v_blk, float* q_pool,
                                            float* k_pool, bsa_stream_t stream) {
  if (sh == nullptr) {
    t_detail.clear();
    return fail(BSA_ERR_INVALID_ARG, "shard description is required");
  }
  const void* const* xsh[3] = {q_shards, k_shards, v_shards};
  return prologue_impl(gi, frames, t_offset, sh, xsh, gamma_q, gamma_k, eps, rope_theta, q_blk,
                       k_blk, v_blk, q_pool, k_pool, stream);
}

static bsa_status_t prologue_bwd_impl(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                      const bsa_shards_t* sd, const void* const* const xsh[2],
                                      const float* gamma_q, const float* gamma_k, float eps,
                                      float rope_theta, const void* dq_blk, const void* dk_blk,
                                      const void* dv_blk, void* const* const dxsh[3],
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
  RasterShards sh;
  if ((st = make_shards(g, frames, sd, &sh)) != BSA_OK) return st;
  const void* dz[3] = {dq_blk, dk_blk, dv_blk};
  const float* gams[2] = {gamma_q, gamma_k};
  float* dgs[2] = {dgamma_q, dgamma_k};
  bool any = false, any_gain = false;
  for (int i = 0; i < 3; ++i) {
    if ((dz[i] == nullptr) != (dxsh[i] == nullptr))
      return fail(BSA_ERR_INVALID_ARG, "gradient %d and its output must both be given or both NULL", i);
    if (dz[i] && (!aligned(dz[i], 16) ||
                  !shard_ptrs_ok(reinterpret_cast<const void* const*>(dxsh[i]), sh.n)))
      return fail(BSA_ERR_INVALID_ARG, "tensor %d: a shard is NULL or a tensor is not 16-byte aligned", i);
    any |= dz[i] != nullptr;
  }
  if (!any) return fail(BSA_ERR_INVALID_ARG, "no tensor to process");
  for (int i = 0; i < 2; ++i) {
    if (dz[i] && gams[i]) {
      if (!xsh[i] || !dgs[i])
        return fail(BSA_ERR_INVALID_ARG, "with a gain, tensor %d needs its raster input and a dgamma output", i);
      if (!shard_ptrs_ok(xsh[i], sh.n))
        return fail(BSA_ERR_INVALID_ARG, "raster input %d: a shard is NULL or not 16-byte aligned", i);
      any_gain = true;
    }
  }
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
  f.sh = sh;
  for (int i = 0; i < 3; ++i) {
    for (int s2 = 0; s2 < kMaxShards; ++s2) f.x[i][s2] = nullptr;
    f.y[i] = nullptr;
  }
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
    for (int s2 = 0; s2 < kMaxShards; ++s2)
      a.dx[i][s2] = (dxsh[i] && s2 < sh.n) ? static_cast<__nv_bfloat16*>(dxsh[i][s2]) : nullptr;
  }
  for (int i = 0; i < 2; ++i) {
    const bool gain = dz[i] && gams[i];
    for (int s2 = 0; s2 < kMaxShards; ++s2)
      a.x[i][s2] = (gain && s2 < sh.n) ? static_cast<const __nv_bfloat16*>(xsh[i][s2]) : nullptr;
    a.part[i] = gain ? reinterpret_cast<float*>(static_cast<char*>(ws) + i * part_bytes) : nullptr;
    if (!gain) dgs[i] = nullptr;
  }
  cudaError_t e = launch_prologue_bwd(a, dgs, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "prologue backward launch");
  return BSA_OK;
}

bsa_status_t rope3d_qknorm_prologue_bwd(const bsa_geom_t* gi, int32_t frames, int32_t t_offset,
                                        const void* q_raster, const void* k_raster,
                                        const float* gamma_q, const float* gamma_k, float eps,
                                        float rope_theta, const void* dq_blk, const void* dk_blk,
                                        const void* dv_blk, void* dq, void* dk, void* dv,
                                        float* dgamma_q, float* dgamma_k, void* ws, size_t ws_bytes,
                                        bsa_stream_t stream) {
  const void* xone[2][1] = {{q_raster}, {k_raster}};
  const void* const* xsh[2] = {q_raster ? xone[0] : nullptr, k_raster ? xone[1] : nullptr};
  void* done[3][1] = {{dq}, {dk}, {dv}};
  void* const* dxsh[3] = {dq ? done[0] : nullptr, dk ? done[1] : nullptr, dv ? done[2] : nullptr};
  return prologue_bwd_impl(gi, frames, t_offset, nullptr, xsh, gamma_q, gamma_k, eps, rope_theta,
                           dq_blk, dk_blk, dv_blk, dxsh, dgamma_q, dgamma_k, ws, ws_bytes, stream);
}

bsa_status_t rope3d_qknorm_prologue_bwd_sharded(
    const bsa_geom_t* gi, int32_t frames, int32_t t_offset, const bsa_shards_t* sh,
    const void* const* q_shards, const void* const* k_shards, const float* gamma_q,
    const float* gamma_k, float eps, float rope_theta, const void* dq_blk, const void* dk_blk,
    const void* dv_blk, void* const* dq_shards, void* const* dk_shards, void* const* dv_shards,
    float* dgamma_q, float* dgamma_k, void* ws, size_t ws_bytes, bsa_stream_t stream) {
  if (sh == nullptr) {
    t_detail.clear();
    return fail(BSA_ERR_INVALID_ARG, "shard description is required");
  }
  const void* const* xsh[2] = {q_shards, k_shards};
  void* const* dxsh[3] = {dq_shards, dk_shards, dv_shards};
  return prologue_bwd_impl(gi, frames, t_offset, sh, xsh, gamma_q, gamma_k, eps, rope_theta,
                           dq_blk, dk_blk, dv_blk, dxsh, dgamma_q, dgamma_k, ws, ws_bytes, stream);
}

bsa_status_t bsa_blocked_to_raster_sharded(const bsa_geom_t* gi, int32_t frames,
                                           const bsa_shards_t* sh, const void* x_blk,
                                           void* const* x_shards, bsa_stream_t stream) {
  if (sh == nullptr || x_blk == nullptr || x_shards == nullptr) {
    t_detail.clear();
    return fail(BSA_ERR_INVALID_ARG, "shard description, x_blk and x_shards are required");
  }
  const void* const* xsh[2] = {nullptr, nullptr};
  void* const* dxsh[3] = {nullptr, nullptr, x_shards};
  return prologue_bwd_impl(gi, frames, 0, sh, xsh, nullptr, nullptr, 0.f, 0.f, nullptr, nullptr,
                           x_blk, dxsh, nullptr, nullptr, nullptr, 0, stream);
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

bsa_status_t bsa_kernel_time_stats(int32_t* launches, float* total_ms, float* min_ms,
                                   float* median_ms) {
  t_detail.clear();
  if (!launches || !total_ms) return fail(BSA_ERR_INVALID_ARG, "launches and total_ms are required");
  KernelTimer& t = kernel_timer();
  std::lock_guard<std::mutex> lk(t.mu);
  bsa_status_t st = BSA_OK;
  std::vector<float> each;
  for (int k = 0; k < kNumTimed; ++k) {
    launches[k] = 0;
    total_ms[k] = 0.f;
    each.clear();
    for (auto& pr : t.pending[k]) {
      float ms = 0.f;
      cudaError_t e = cudaEventSynchronize(pr.second);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, pr.first, pr.second);
      if (e != cudaSuccess && st == BSA_OK) st = cuda_fail(e, "kernel timing event");
      ++launches[k];
      total_ms[k] += ms;
      each.push_back(ms);
      t.pool.push_back(pr.first);
      t.pool.push_back(pr.second);
    }
    t.pending[k].clear();
    std::sort(each.begin(), each.end());
    const size_t n = each.size();
    if (min_ms) min_ms[k] = n ? each[0] : 0.f;
    if (median_ms) median_ms[k] = n ? (n % 2 ? each[n / 2] : 0.5f * (each[n / 2 - 1] + each[n / 2])) : 0.f;
  }
  return st;
}

bsa_status_t bsa_kernel_times(int32_t* launches, float* total_ms) {
  return bsa_kernel_time_stats(launches, total_ms, nullptr, nullptr);
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

// ---------------------------------------------------------------- CUDA IPC of shard buffers
// A handle is the cudaIpcMemHandle of the allocation holding the pointer followed by the
// pointer's byte offset in it (the caching allocators above the library hand out pieces of
// larger allocations).  Imported mappings are remembered so that bsa_ipc_close can unmap the
// allocation base.
namespace {
typedef CUresult (*AddressRangeFn)(CUdeviceptr*, size_t*, CUdeviceptr);
struct IpcHandle {
  cudaIpcMemHandle_t mem;
  uint64_t offset;
};
static_assert(sizeof(IpcHandle) <= BSA_IPC_HANDLE_BYTES, "IPC handle size");
struct IpcMapping {
  cudaIpcMemHandle_t mem;
  void* base;
  int refs;
};
std::mutex g_ipc_mu;
std::vector<IpcMapping> g_ipc_bases;              // one mapping per peer allocation
std::vector<std::pair<void*, void*>> g_ipc_maps;  // (imported pointer, mapped base), per import

AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(f);
  });
  return fn;
}
}  // namespace

bsa_status_t bsa_ipc_export(const void* dev_ptr, void* handle) {
  t_detail.clear();
  if (!dev_ptr || !handle) return fail(BSA_ERR_INVALID_ARG, "dev_ptr and handle are required");
  AddressRangeFn range = address_range_fn();
  if (!range) return fail(BSA_ERR_CUDA, "cuMemGetAddressRange is not available");
  CUdeviceptr base = 0;
  size_t bytes = 0;
  if (range(&base, &bytes, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return fail(BSA_ERR_INVALID_ARG, "dev_ptr is not device memory of this process");
  IpcHandle h;
  std::memset(&h, 0, sizeof(h));
  cudaError_t e = cudaIpcGetMemHandle(&h.mem, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return cuda_fail(e, "cudaIpcGetMemHandle");
  h.offset = reinterpret_cast<uintptr_t>(dev_ptr) - static_cast<uintptr_t>(base);
  std::memset(handle, 0, BSA_IPC_HANDLE_BYTES);
  std::memcpy(handle, &h, sizeof(h));
  return BSA_OK;
}

bsa_status_t bsa_ipc_import(const void* handle, void** dev_ptr) {
  t_detail.clear();
  if (!handle || !dev_ptr) return fail(BSA_ERR_INVALID_ARG, "handle and dev_ptr are required");
  IpcHandle h;
  std::memcpy(&h, handle, sizeof(h));
  std::lock_guard<std::mutex> lk(g_ipc_mu);
  void* base = nullptr;
  for (IpcMapping& m : g_ipc_bases)  // an allocation is mapped once per process
    if (std::memcmp(&m.mem, &h.mem, sizeof(h.mem)) == 0) {
      base = m.base;
      ++m.refs;
      break;
    }
  if (!base) {
    cudaError_t e = cudaIpcOpenMemHandle(&base, h.mem, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(e, "cudaIpcOpenMemHandle");
    g_ipc_bases.push_back(IpcMapping{h.mem, base, 1});
  }
  void* p = static_cast<char*>(base) + h.offset;
  g_ipc_maps.emplace_back(p, base);
  *dev_ptr = p;
  return BSA_OK;
}

bsa_status_t bsa_ipc_close(void* dev_ptr) {
  t_detail.clear();
  std::lock_guard<std::mutex> lk(g_ipc_mu);
  void* base = nullptr;
  for (size_t k = 0; k < g_ipc_maps.size(); ++k)
    if (g_ipc_maps[k].first == dev_ptr) {
      base = g_ipc_maps[k].second;
      g_ipc_maps.erase(g_ipc_maps.begin() + (long)k);
      break;
    }
  if (!base) return fail(BSA_ERR_INVALID_ARG, "pointer was not imported by bsa_ipc_import");
  for (size_t k = 0; k < g_ipc_bases.size(); ++k)
    if (g_ipc_bases[k].base == base && --g_ipc_bases[k].refs == 0) {
      g_ipc_bases.erase(g_ipc_bases.begin() + (long)k);
      cudaError_t e = cudaIpcCloseMemHandle(base);
      if (e != cudaSuccess) return cuda_fail(e, "cudaIpcCloseMemHandle");
      break;
    }
  return BSA_OK;
}

#include "route_noalloc.cu"
