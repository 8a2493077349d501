// route.cu -- block pooling, block scores and top-r selection (BSA routing).
//
// Sources: "LongCat-Video : Generate 1 minute long AI videos with this model", section
// "Sparse attention" (split the tokens into small 3D cubes; each cube looks only at the few
// most relevant ones, chosen by similarity); "LongCat-Video视频生成模型发布 迈出世界模型探索
// 第一步", section 块稀疏注意力（BSA） (only the top-r key blocks are computed).
//
// pool_kernel      : qbar/kbar = mean over the valid tokens of each block (fp32); the sum and
//                    channel-wise max are the pooling variants.
// score_select     : s_ij = qbar_i . kbar_j in fp32 on CUDA cores (ranking needs fp32, the
//                    work is ~NBq*NBk*D FMAs per head, tiny next to the attention), masked
//                    to -inf by the block-causal rule (causal chunks and / or the two-segment
//                    conditioning form), then an exact warp-level radix select
//                    of the top r per row on order-preserving 32-bit keys, ties resolved to
//                    the lower block index, emitted in ascending block order.
// Variants (the pages leave the routing rule open): the own key block NBc + i forced into
// every query block's selection (its score is taken as +inf, so it always ranks first), and
// one selection per (b, query block) shared by all heads, ranked by the score summed over
// the heads, s_ij = sum_h qbar_hi . kbar_hj.
#include "common.cuh"

namespace bsa {

constexpr int kPoolThreads = 256;
constexpr int kPoolMean = 0, kPoolSum = 1, kPoolMax = 2;
constexpr unsigned kRouteForceSelf = 1u, kRouteSharedHeads = 2u;

template <int D, int MODE>  // MODE: kPoolMean, kPoolSum, kPoolMax
__global__ void __launch_bounds__(kPoolThreads)
    pool_kernel(const __nv_bfloat16* __restrict__ x, int frames, int nb, Geo g,
                float* __restrict__ out) {
  constexpr int CPR = D / 8, RG = kPoolThreads / CPR;
  constexpr float kInit = MODE == kPoolMax ? -INFINITY : 0.f;
  __shared__ float red[RG][D];
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, cc = tid % CPR, rg = tid / CPR;
  int vt, vh, vw;
  block_extent(g, frames, blk, vt, vh, vw);
  const __nv_bfloat16* base = x + (((size_t)b * g.H + h) * nb + blk) * (size_t)g.BS * D;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = kInit;
  const int nvalid = max(vt, 0) * max(vh, 0) * max(vw, 0);
  for (int slot = rg; slot < nvalid; slot += RG) {  // valid tokens are the first slots
    {
      const uint4 raw = __ldg(reinterpret_cast<const uint4*>(base + (size_t)slot * D + cc * 8));
      const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(p2[e]);
        if (MODE == kPoolMax) {
          acc[2 * e] = fmaxf(acc[2 * e], f.x); acc[2 * e + 1] = fmaxf(acc[2 * e + 1], f.y);
        } else {
          acc[2 * e] += f.x; acc[2 * e + 1] += f.y;
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][cc * 8 + e] = acc[e];
  __syncthreads();
  for (int d = tid; d < D; d += kPoolThreads) {
    float s = kInit;
    for (int r = 0; r < RG; ++r) s = MODE == kPoolMax ? fmaxf(s, red[r][d]) : s + red[r][d];
    float v = 0.f;
    if (nvalid) v = MODE == kPoolMean ? s / (float)nvalid : s;
    out[(((size_t)b * g.H + h) * nb + blk) * D + d] = v;
  }
}

// ------------------------------------------------------------------------------ scores
constexpr int kSelThreads = 256;
constexpr int kKT = 128;  // key blocks per smem tile

__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f + 0.0f);  // + 0.0f folds -0 into +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelectArgs {
  Geo g;
  int r, qt;                  // top-r, query blocks per CTA
  unsigned flags = 0;         // kRouteForceSelf | kRouteSharedHeads
  const float* qpool;         // [B,H,NBq,D]
  const float* kpool;         // [B,H,NBq,D] current key blocks
  const float* kpool_cache;   // [B,H,NBc,D] or null
  int* idx;                   // [B,H,NBq,r]
  int* cnt;                   // [B,H,NBq]
};

template <int D, int RPT>  // RPT = query rows per thread = qt / 8
__global__ void __launch_bounds__(kSelThreads) score_select_kernel(const SelectArgs a) {
  constexpr int LD = D + 4;  // padded row (floats): conflict-free 16-byte reads
  constexpr int QT = RPT * 8;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* qs = reinterpret_cast<float*>(smem_raw);     // [QT][LD]
  float* ks = qs + QT * LD;                           // [kKT][LD]
  float* sc = ks + kKT * LD;                          // [QT][NBk]
  int* hist = reinterpret_cast<int*>(sc + (size_t)QT * a.g.NBk);  // [8 warps][256]

  const Geo& g = a.g;
  const int i0 = blockIdx.x * QT, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const bool shared_heads = (a.flags & kRouteSharedHeads) != 0;
  const bool force_self = (a.flags & kRouteForceSelf) != 0;
  // heads whose scores are summed: this CTA's head, or all of them (then gridDim.y == 1)
  const int h_lo = shared_heads ? 0 : h, h_hi = shared_heads ? g.H : h + 1;
  const int nq = min(QT, g.NBq - i0);

  const int ti = tid / 32, tj = tid % 32;
  for (int j0 = 0; j0 < g.NBk; j0 += kKT) {
    float acc[RPT][4];
#pragma unroll
    for (int x = 0; x < RPT; ++x)
#pragma unroll
      for (int m = 0; m < 4; ++m) acc[x][m] = 0.f;
    for (int hh = h_lo; hh < h_hi; ++hh) {
      const size_t bh = (size_t)b * g.H + hh;
      __syncthreads();  // the previous head / tile is no longer read
      if (shared_heads || j0 == 0) {
        for (int e = tid; e < QT * (D / 4); e += kSelThreads) {
          const int ii = e / (D / 4), d4 = e % (D / 4);
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (ii < nq) v = *reinterpret_cast<const float4*>(a.qpool + (bh * g.NBq + i0 + ii) * D + d4 * 4);
          *reinterpret_cast<float4*>(qs + ii * LD + d4 * 4) = v;
        }
      }
      for (int e = tid; e < kKT * (D / 4); e += kSelThreads) {
        const int jj = e / (D / 4), d4 = e % (D / 4), j = j0 + jj;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (j < g.NBc)
          v = *reinterpret_cast<const float4*>(a.kpool_cache + (bh * g.NBc + j) * D + d4 * 4);
        else if (j < g.NBk)
          v = *reinterpret_cast<const float4*>(a.kpool + (bh * g.NBq + (j - g.NBc)) * D + d4 * 4);
        *reinterpret_cast<float4*>(ks + jj * LD + d4 * 4) = v;
      }
      __syncthreads();
#pragma unroll 4
      for (int d = 0; d < D; d += 4) {
        float4 kv[4], qv[RPT];
#pragma unroll
        for (int m = 0; m < 4; ++m) kv[m] = *reinterpret_cast<const float4*>(ks + (tj + 32 * m) * LD + d);
#pragma unroll
        for (int x = 0; x < RPT; ++x) qv[x] = *reinterpret_cast<const float4*>(qs + (ti * RPT + x) * LD + d);
#pragma unroll
        for (int x = 0; x < RPT; ++x)
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            acc[x][m] = fmaf(qv[x].x, kv[m].x, acc[x][m]);
            acc[x][m] = fmaf(qv[x].y, kv[m].y, acc[x][m]);
            acc[x][m] = fmaf(qv[x].z, kv[m].z, acc[x][m]);
            acc[x][m] = fmaf(qv[x].w, kv[m].w, acc[x][m]);
          }
      }
    }
#pragma unroll
    for (int x = 0; x < RPT; ++x) {
      const int ii = ti * RPT + x, i = i0 + ii;
      if (ii >= nq) continue;
      const bool masked = g.chunk || g.cond;
      const int ci = masked ? frame_segment(g, query_block_t0(g, i)) : 0;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int j = j0 + tj + 32 * m;
        if (j >= g.NBk) continue;
        bool ok = true;
        if (masked) ok = frame_segment(g, key_block_t0(g, j)) <= ci;
        // a key block always holds >= 1 valid token when the grid is padded to whole blocks;
        // the own block (same frames, so never masked) ranks above every finite score
        float v = ok ? acc[x][m] : -INFINITY;
        if (force_self && j == g.NBc + i) v = INFINITY;
        sc[(size_t)ii * g.NBk + j] = v;
      }
    }
  }
  __syncthreads();

  // ------------------------------------------------------------ warp radix select per row
  int* hw = hist + warp * 256;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int ii = warp; ii < nq; ii += 8) {
    const float* srow = sc + (size_t)ii * g.NBk;
    int nfin = 0;
    for (int j = lane; j < g.NBk; j += 32) nfin += (srow[j] > -INFINITY) ? 1 : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nfin += __shfl_xor_sync(0xffffffffu, nfin, o);
    const int reff = min(a.r, nfin);
    uint32_t prefix = 0, pmask = 0;
    int k = reff;  // rank (from the top, 1-based) of the threshold key among the candidates
    if (reff > 0) {
      for (int shift = 24; shift >= 0; shift -= 8) {
        for (int e = lane; e < 256; e += 32) hw[e] = 0;
        __syncwarp();
        for (int j = lane; j < g.NBk; j += 32) {
          const float s = srow[j];
          if (s > -INFINITY) {
            const uint32_t key = ordered_key(s);
            if ((key & pmask) == prefix) atomicAdd(&hw[(key >> shift) & 255u], 1);
          }
        }
        __syncwarp();
        int c[8], lsum = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) { c[e] = hw[255 - 8 * lane - e]; lsum += c[e]; }
        int incl = lsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        const int excl = incl - lsum;
        const unsigned hit = __ballot_sync(0xffffffffu, excl < k && k <= incl);
        const int src = __ffs(hit) - 1;
        int bin = 0, above = 0;
        if (lane == src) {
          int cum = excl;
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            if (cum + c[e] >= k) { bin = 255 - 8 * lane - e; above = cum; break; }
            cum += c[e];
          }
        }
        bin = __shfl_sync(0xffffffffu, bin, src);
        above = __shfl_sync(0xffffffffu, above, src);
        prefix |= (uint32_t)bin << shift;
        pmask |= 0xFFu << shift;
        k -= above;
        __syncwarp();
      }
    }
    // emit ascending: keys above the threshold, then the first k keys equal to it
    int written = 0, eq_seen = 0;
    if (reff > 0) {
      for (int base = 0; base < g.NBk; base += 32) {
        const int j = base + lane;
        bool gt = false, eq = false;
        if (j < g.NBk) {
          const float s = srow[j];
          if (s > -INFINITY) {
            const uint32_t key = ordered_key(s);
            gt = key > prefix;
            eq = key == prefix;
          }
        }
        const unsigned eqm = __ballot_sync(0xffffffffu, eq);
        const bool take = gt || (eq && eq_seen + __popc(eqm & lt_mask) < k);
        const unsigned tm = __ballot_sync(0xffffffffu, take);
        const int pos = written + __popc(tm & lt_mask);
        if (take && pos < a.r)
          for (int hh = h_lo; hh < h_hi; ++hh)
            a.idx[(((size_t)b * g.H + hh) * g.NBq + i0 + ii) * a.r + pos] = j;
        written += __popc(tm);
        eq_seen += __popc(eqm);
      }
    }
    written = min(written, a.r);
    for (int hh = h_lo; hh < h_hi; ++hh) {
      const size_t row = ((size_t)b * g.H + hh) * g.NBq + i0 + ii;
      for (int e = written + lane; e < a.r; e += 32) a.idx[row * a.r + e] = -1;
      if (lane == 0) a.cnt[row] = written;
    }
  }
}

template <int D>
static cudaError_t launch_pool_d(const __nv_bfloat16* x, int frames, int nb, const Geo& g,
                                 int mode, float* out, cudaStream_t s) {
  dim3 grid(nb, g.H, g.B);
  if (mode == kPoolSum) pool_kernel<D, kPoolSum><<<grid, kPoolThreads, 0, s>>>(x, frames, nb, g, out);
  else if (mode == kPoolMax) pool_kernel<D, kPoolMax><<<grid, kPoolThreads, 0, s>>>(x, frames, nb, g, out);
  else pool_kernel<D, kPoolMean><<<grid, kPoolThreads, 0, s>>>(x, frames, nb, g, out);
  return cudaGetLastError();
}

cudaError_t launch_pool(const __nv_bfloat16* x, int frames, int nb, const Geo& g, float* out,
                        cudaStream_t s, int mode = kPoolMean) {
  return g.D == 128 ? launch_pool_d<128>(x, frames, nb, g, mode, out, s)
                    : launch_pool_d<64>(x, frames, nb, g, mode, out, s);
}

// query rows per CTA: the largest of 32 / 16 / 8 whose tiles and score rows (QT * NBk * 4
// bytes) fit the 227 KB of shared memory a CTA may have; 0 if none does
int select_rows_per_cta(const Geo& g) {
  for (int qt : {32, 16, 8}) {
    size_t bytes = (size_t)(qt + kKT) * (g.D + 4) * 4 + (size_t)qt * g.NBk * 4 + 8 * 256 * 4;
    if (bytes <= 227 * 1024) return qt;
  }
  return 0;
}

size_t select_smem_bytes(const Geo& g, int qt) {
  return (size_t)(qt + kKT) * (g.D + 4) * 4 + (size_t)qt * g.NBk * 4 + 8 * 256 * 4;
}

template <int D, int RPT>
static cudaError_t launch_sel_t(const SelectArgs& a, cudaStream_t s) {
  const Geo& g = a.g;
  dim3 grid((g.NBq + a.qt - 1) / a.qt, (a.flags & kRouteSharedHeads) ? 1 : g.H, g.B);
  size_t smem = select_smem_bytes(g, a.qt);
  cudaError_t e = cudaFuncSetAttribute(score_select_kernel<D, RPT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  score_select_kernel<D, RPT><<<grid, kSelThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_select(const SelectArgs& a, cudaStream_t s) {
  const int rpt = a.qt / 8;
  if (a.g.D == 128) {
    if (rpt == 4) return launch_sel_t<128, 4>(a, s);
    if (rpt == 2) return launch_sel_t<128, 2>(a, s);
    return launch_sel_t<128, 1>(a, s);
  }
  if (rpt == 4) return launch_sel_t<64, 4>(a, s);
  if (rpt == 2) return launch_sel_t<64, 2>(a, s);
  return launch_sel_t<64, 1>(a, s);
}

}  // namespace bsa
