// route_noalloc.cu -- bsa_route_noalloc: routing without caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they route: a serving
// engine that reserved the whole device at start-up and hands out nothing else, a host
// framework whose allocator owns every byte, or a latency-critical path where cudaMalloc
// could synchronise the device.  For them this entry point takes only inputs and outputs;
// the block means it needs live in a fixed array inside the library.
//
// The array is a file-scope __device__ array of kNoallocScratchBytes (16 MiB).  Every GPU
// that loads the library holds it until the process exits.  Host code cannot pass the
// array's name to a kernel (on the host it is only a stand-in symbol), so the first call on
// each device looks up its device address with cudaGetSymbolAddress, with that device
// current, and caches it; make that first call before any stream capture.  The cache keeps
// the CUDA context the address belongs to: after cudaDeviceReset (or any re-creation of the
// device's primary context) the next call finds a different context and looks the address up
// again, in the new context, rather than launching on a stale one.  All calls share
// the array: two calls whose work overlaps on the GPU (different streams, no ordering
// between them) race on it.  Nothing in it needs to start at zero: the pooling kernel
// overwrites every mean it later reads.
//
// This file is included by bsa_lib.cu (single translation unit) after the host helpers.

namespace bsa {

constexpr size_t kNoallocScratchBytes = 16u << 20;
static __device__ __align__(256) unsigned char g_route_scratch[kNoallocScratchBytes];

namespace {
constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoallocMaxDevices] = {nullptr};
CUcontext g_noalloc_ctx[kNoallocMaxDevices] = {nullptr};  // context each address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn g_ctx_get = nullptr;
std::once_flag g_ctx_get_once;

// The calling thread's current CUDA context (nullptr if none is bound yet or the driver entry
// point is unavailable; a null context never matches a cached one, so it forces a lookup).
CUcontext current_ctx() {
  std::call_once(g_ctx_get_once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  CUcontext c = nullptr;
  if (g_ctx_get && g_ctx_get(&c) != CUDA_SUCCESS) c = nullptr;
  return c;
}
}  // namespace

}  // namespace bsa

extern "C" BSA_API bsa_status_t bsa_route_noalloc(const bsa_geom_t* gi, int32_t top_r,
                                                  const void* q_blk, const void* k_blk,
                                                  const float* kpool_cache, int32_t* idx,
                                                  int32_t* cnt, bsa_stream_t stream) {
  using namespace bsa;
  t_detail.clear();
  Geo g;
  bsa_status_t st = make_geo(gi, &g);
  if (st != BSA_OK) return st;
  if (top_r < 1) return fail(BSA_ERR_INVALID_ARG, "top_r must be >= 1");
  if (!q_blk || !k_blk || !idx || !cnt)
    return fail(BSA_ERR_INVALID_ARG, "q_blk, k_blk, idx and cnt are required");
  if (g.NBc > 0 && !kpool_cache)
    return fail(BSA_ERR_INVALID_ARG, "kpool_cache is required when cached_t > 0");
  const void* ptrs[3] = {q_blk, k_blk, kpool_cache};
  for (const void* p : ptrs)
    if (p && !aligned(p, 16)) return fail(BSA_ERR_INVALID_ARG, "inputs must be 16-byte aligned");
  const RouteWs w = route_ws(g);
  if (select_rows_per_cta(g) == 0)
    return fail(BSA_ERR_UNSUPPORTED, "%d key blocks do not fit the select kernel", g.NBk);
  if (w.total > kNoallocScratchBytes)
    return fail(BSA_ERR_UNSUPPORTED,
                "bsa_route_noalloc needs %zu scratch bytes but holds %zu (B*H*NBq*D*8 must not "
                "exceed it); use bsa_route with a caller workspace",
                w.total, kNoallocScratchBytes);
  int n_sm = 0;
  st = check_device(&n_sm);
  if (st != BSA_OK) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoallocMaxDevices)
    return fail(BSA_ERR_UNSUPPORTED, "device %d is beyond the %d devices bsa_route_noalloc tracks",
                dev, kNoallocMaxDevices);
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    const CUcontext ctx = current_ctx();
    if (g_noalloc_ptr[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_route_scratch);  // this device is current
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(route scratch)");
      g_noalloc_ptr[dev] = ptr;
      g_noalloc_ctx[dev] = current_ctx();  // the lookup has bound the device's context
    }
    scratch = g_noalloc_ptr[dev];
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* qpool = reinterpret_cast<float*>(static_cast<char*>(scratch) + w.qpool);
  float* kpool = reinterpret_cast<float*>(static_cast<char*>(scratch) + w.kpool);
  if ((e = launch_pool(static_cast<const __nv_bfloat16*>(q_blk), g.T, g.NBq, g, qpool, s)) != cudaSuccess)
    return cuda_fail(e, "pool launch");
  if ((e = launch_pool(static_cast<const __nv_bfloat16*>(k_blk), g.T, g.NBq, g, kpool, s)) != cudaSuccess)
    return cuda_fail(e, "pool launch");
  SelectArgs a;
  a.g = g;
  a.r = top_r;
  a.qt = select_rows_per_cta(g);
  a.qpool = qpool;
  a.kpool = kpool;
  a.kpool_cache = kpool_cache;
  a.idx = idx;
  a.cnt = cnt;
  if ((e = launch_select(a, s)) != cudaSuccess) return cuda_fail(e, "select launch");
  return BSA_OK;
}
