// cache_append.cu -- continuation caches for the next round.
//
// Source: "LongCat-Video 高效長視頻生成探索世界模型的第壹步", section 2.1 (Block-Causal attention
// lets the frames already produced be cached and reused), and "LongCat-Video : Generate 1
// minute long AI videos with this model", section "The core idea" (the fixed conditioning
// frames are not reprocessed).  After a round over t_frames current frames, the cache for the
// next round holds the old cached frames followed by this round's frames: per (b, h) the
// blocked K and V (and the fp32 key-block means used by routing) are the old cache's NBc
// blocks then the current NBq blocks.  Keys were rotated with absolute frame positions, so
// they are reused as they are.  A plain vectorised copy (HBM-bound).
#include <algorithm>

#include "common.cuh"

namespace bsa {

// dst[bh][j] = j < nc ? c[bh][j] : x[bh][j - nc], rows of `row` 16-byte vectors
__global__ void __launch_bounds__(256) cache_append_kernel(const uint4* __restrict__ c,
                                                           const uint4* __restrict__ x,
                                                           uint4* __restrict__ dst, int bh_n,
                                                           int nc, int nx, int row) {
  const size_t per_bh = (size_t)(nc + nx) * row;
  const size_t total = (size_t)bh_n * per_bh;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const size_t bh = e / per_bh, r = e % per_bh;
    const size_t j = r / row, k = r % row;
    dst[e] = j < (size_t)nc ? c[(bh * nc + j) * row + k] : x[(bh * nx + (j - nc)) * row + k];
  }
}

cudaError_t launch_cache_append(const void* c, const void* x, void* dst, int bh_n, int nc, int nx,
                                size_t row_bytes, int n_sm, cudaStream_t s) {
  const int row = (int)(row_bytes / 16);
  const size_t total = (size_t)bh_n * (nc + nx) * row;
  const int blocks = (int)std::min<size_t>((total + 255) / 256, (size_t)n_sm * 8);
  cache_append_kernel<<<blocks > 0 ? blocks : 1, 256, 0, s>>>(
      static_cast<const uint4*>(c), static_cast<const uint4*>(x), static_cast<uint4*>(dst), bh_n,
      nc, nx, row);
  return cudaGetLastError();
}

}  // namespace bsa
