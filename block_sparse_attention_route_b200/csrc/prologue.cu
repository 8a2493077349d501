// prologue.cu -- fused QK-RMSNorm + 3D RoPE + raster -> blocked relayout (+ block means).
//
// Source: "美团LongCat-Video揭秘：13.6B参数长视频生成模型如何终结画面漂移？", section 三 模型架构
// (the DiT uses 3D RoPE position encoding and RMSNorm + QKNorm).  The RoPE channel split and
// pairing, the norm placement (before RoPE) and eps are this library's documented readings.
//
// HBM-bound: every (token, head) row of q, k, v is read once (D bf16) and written once to
// its slot of the blocked layout (a block's valid tokens first, see slot_local); pad slots
// are written as zeros.  One CTA handles one
// block of the padded grid for 8 heads; D/8 lanes own one row (16-byte vectors).  Rows are
// visited slot-major, head-minor, so consecutive row groups read consecutive heads of one
// token (a contiguous 8 x D x 2-byte run of the raster) and every lane keeps one head.
// The cos/sin table of the block's (t, h, w) positions is built once per CTA in shared
// memory (fp64 angles).
#include "common.cuh"

namespace bsa {

// Raster tensors may be split along frames into shards (one per rank of a sequence-parallel
// group, each possibly on another GPU): shard s holds frames [s * frames, (s + 1) * frames)
// of the grid as [B, frames * GH * GW, h_stride, D], and this call processes raster heads
// h0 .. h0 + g.H - 1 of it.  One shard with h_stride = g.H and h0 = 0 is the plain layout.
// Reading or writing the shards of other ranks through their pointers is the sequence <->
// head exchange of Ulysses parallelism, fused into the relayout.
constexpr int kMaxShards = 8;
struct RasterShards {
  int n, frames;     // shards, frames per shard
  int h_stride, h0;  // heads of every raster row, first head processed
};

// Element offset of (b, frame t of the grid, row hh, column ww, head h, channel c0) in its
// shard, and the shard s.  kSharded = false (every single-GPU call: one shard, all heads)
// compiles to the plain raster offset.
// n_raster: tokens of the plain tensor (frames * GH * GW).
template <bool kSharded, int D>
__device__ __forceinline__ size_t shard_elem(const RasterShards& sh, const Geo& g, size_t n_raster,
                                             int b, int t, int hh, int ww, int h, int c0, int& s) {
  if constexpr (!kSharded) {
    s = 0;
    const size_t n = ((size_t)t * g.GH + hh) * g.GW + ww;
    return (((size_t)b * n_raster + n) * g.H + h) * D + c0;
  } else {
    s = t / sh.frames;
    const size_t n = ((size_t)(t - s * sh.frames) * g.GH + hh) * g.GW + ww;
    const size_t per_shard = (size_t)sh.frames * g.GH * g.GW;
    return (((size_t)b * per_shard + n) * sh.h_stride + sh.h0 + h) * D + c0;
  }
}

struct PrologueArgs {
  Geo g;
  int frames, t_offset, nbt;  // grid being processed: frames, RoPE frame offset, t-blocks
  RasterShards sh;
  const __nv_bfloat16* x[3][kMaxShards];  // raster inputs per shard (x[w][0] == NULL: skip)
  __nv_bfloat16* y[3];
  const float* gamma[2];
  float* pool[2];
  float eps, theta;
  int dt, dh, dw;  // RoPE axis widths (channels)
};

constexpr int kPrologueThreads = 256;
constexpr int kHeadsPerCta = 8;

// cos/sin of every RoPE angle a block needs, in fp64 then rounded: axis t rows [0, bt), h
// rows after, w rows last; each row holds that axis' pairs (pos * theta^(-2i/width)).
__device__ void build_rope_table(const PrologueArgs& a, int ibt, int ibh, int ibw, float2* tab) {
  const Geo& g = a.g;
  const int pt = a.dt / 2, ph = a.dh / 2, pw = a.dw / 2;
  const int off_h = g.bt * pt, off_w = off_h + g.bh * ph, ntab = off_w + g.bw * pw;
  for (int e = threadIdx.x; e < ntab; e += blockDim.x) {
    int pos, i, width;
    if (e < off_h) {
      pos = a.t_offset + ibt * g.bt + e / pt; i = e % pt; width = a.dt;
    } else if (e < off_w) {
      int r = e - off_h; pos = ibh * g.bh + r / ph; i = r % ph; width = a.dh;
    } else {
      int r = e - off_w; pos = ibw * g.bw + r / pw; i = r % pw; width = a.dw;
    }
    double ang = (double)pos * pow((double)a.theta, -2.0 * (double)i / (double)width);
    double s, c;
    sincos(ang, &s, &c);
    tab[e] = make_float2((float)c, (float)s);
  }
}

template <int D, bool kSharded>
__global__ void __launch_bounds__(kPrologueThreads)
    prologue_kernel(const PrologueArgs a) {
  constexpr int LPR = D / 8;                     // lanes per row
  constexpr int RPP = kPrologueThreads / LPR;    // rows per pass
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* pool_s = reinterpret_cast<float*>(smem_raw);            // [2][8][D]
  float2* tab = reinterpret_cast<float2*>(pool_s + 2 * kHeadsPerCta * D);

  const Geo& g = a.g;
  const int blk = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int per_t = g.nbh * g.nbw;
  const int ibt = blk / per_t, ibh = (blk % per_t) / g.nbw, ibw = blk % g.nbw;
  int vt, vh, vw;
  block_extent(g, a.frames, blk, vt, vh, vw);
  const int nvalid = max(vt, 0) * max(vh, 0) * max(vw, 0);
  const bool full = vh == g.bh && vw == g.bw;  // slot decode by shifts
  const bool rope = a.theta > 0.f;

  // ---- cos/sin table: axis t rows [0,bt), h rows [bt, bt+bh), w rows after; each row
  //      holds that axis' pairs.
  const int pt = a.dt / 2, ph = a.dh / 2, pw = a.dw / 2;
  const int off_h = g.bt * pt, off_w = off_h + g.bh * ph;
  if (rope) build_rope_table(a, ibt, ibh, ibw, tab);
  for (int e = tid; e < 2 * kHeadsPerCta * D; e += kPrologueThreads) pool_s[e] = 0.f;
  __syncthreads();

  const int rid = tid / LPR, cl = tid % LPR, c0 = cl * 8;
  const int heads_here = min(kHeadsPerCta, g.H - hg * kHeadsPerCta);
  // (slot, head) pairs, head fastest.  A sharded call (a rank's slice of the heads, often
  // fewer than 8) spreads its rows over the heads present; the plain path keeps the constant
  // stride and skips the missing heads of a last, partial group.
  const int hpc = kSharded ? heads_here : kHeadsPerCta;
  const int rows = hpc * g.BS;
  const size_t n_raster = (size_t)a.frames * g.GH * g.GW;

  // RoPE coordinates of this lane's 4 channel pairs: axis (0 t, 1 h, 2 w) and pair index.
  int ax[4], pi[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    int p = c0 / 2 + q;
    if (2 * p < a.dt) { ax[q] = 0; pi[q] = p; }
    else if (2 * p < a.dt + a.dh) { ax[q] = 1; pi[q] = p - pt; }
    else { ax[q] = 2; pi[q] = p - pt - ph; }
  }

  for (int which = 0; which < 3; ++which) {
    __nv_bfloat16* __restrict__ y = a.y[which];
    const __nv_bfloat16* __restrict__ x0 = a.x[which][0];  // the one shard of a plain call
    if (x0 == nullptr) continue;
    const bool qk = which < 2;
    const float* gam = qk ? a.gamma[which] : nullptr;
    const bool do_rope = qk && rope;
    const bool do_pool = qk && a.pool[which] != nullptr;
    float gv[8];
    if (gam) {
#pragma unroll
      for (int e = 0; e < 8; ++e) gv[e] = gam[c0 + e];
    }
    float psum[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    int cur_h = -1;
    // this lane's 16 bytes of the row of pass `bs` (zero for pad slots and absent heads); the
    // next pass's load is issued before the current pass is processed, so two are in flight
    auto fetch = [&](int bs) -> uint4 {
      const int row = bs + rid;
      const int hl = row % hpc, slot = row / hpc;
      uint4 r = make_uint4(0u, 0u, 0u, 0u);
      if (row < rows && hl < heads_here && slot < nvalid) {
        int lt, lh, lw;
        slot_local(g, slot, vh, vw, full, lt, lh, lw);
        const int t = ibt * g.bt + lt, hh = ibh * g.bh + lh, ww = ibw * g.bw + lw;
        int sidx;
        const size_t off = shard_elem<kSharded, D>(a.sh, g, n_raster, b, t, hh, ww,
                                                   hg * kHeadsPerCta + hl, c0, sidx);
        r = __ldg(reinterpret_cast<const uint4*>((kSharded ? a.x[which][sidx] : x0) + off));
      }
      return r;
    };
    uint4 nxt = fetch(0);
    for (int base = 0; base < rows; base += RPP) {
      const uint4 raw = nxt;
      if (base + RPP < rows) nxt = fetch(base + RPP);
      const int row = base + rid;
      const int hl = row % hpc, slot = row / hpc;
      const bool in = row < rows && hl < heads_here;
      const int h = hg * kHeadsPerCta + hl;
      const bool valid = in && slot < nvalid;
      int lt = 0, lh = 0, lw = 0;
      if (valid) slot_local(g, slot, vh, vw, full, lt, lh, lw);
      float v[8];
      {
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(p2[e]);
          v[2 * e] = f.x; v[2 * e + 1] = f.y;
        }
      }
      if (gam) {  // RMSNorm over the row: every lane takes part in the shuffles
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(v[e], v[e], ss);
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = rsqrtf(ss * (1.0f / D) + a.eps);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = v[e] * rs * gv[e];
      }
      if (do_rope && valid) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 cs;
          if (ax[q] == 0) cs = tab[lt * pt + pi[q]];
          else if (ax[q] == 1) cs = tab[off_h + lh * ph + pi[q]];
          else cs = tab[off_w + lw * pw + pi[q]];
          const float x0 = v[2 * q], x1 = v[2 * q + 1];
          v[2 * q] = x0 * cs.x - x1 * cs.y;
          v[2 * q + 1] = x0 * cs.y + x1 * cs.x;
        }
      }
      uint4 outv;
      uint32_t* o32 = reinterpret_cast<uint32_t*>(&outv);
#pragma unroll
      for (int e = 0; e < 4; ++e) o32[e] = valid ? pack_bf16x2(v[2 * e], v[2 * e + 1]) : 0u;
      if (in) {
        *reinterpret_cast<uint4*>(
            y + ((((size_t)b * g.H + h) * (size_t)(a.nbt * per_t) + blk) * g.BS + slot) * D +
            c0) = outv;
      }
      if (do_pool && in) {
        if (hl != cur_h) {
          if (cur_h >= 0) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              atomicAdd(&pool_s[(which * kHeadsPerCta + cur_h) * D + c0 + e], psum[e]);
              psum[e] = 0.f;
            }
          }
          cur_h = hl;
        }
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&outv);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(p2[e]);
          psum[2 * e] += f.x; psum[2 * e + 1] += f.y;
        }
      }
    }
    if (do_pool && cur_h >= 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        atomicAdd(&pool_s[(which * kHeadsPerCta + cur_h) * D + c0 + e], psum[e]);
    }
  }
  __syncthreads();
  for (int which = 0; which < 2; ++which) {
    float* out = a.pool[which];
    if (out == nullptr || a.x[which][0] == nullptr) continue;
    const float inv = nvalid > 0 ? 1.0f / (float)nvalid : 0.f;
    for (int e = tid; e < heads_here * D; e += kPrologueThreads) {
      const int hl = e / D, d = e % D, h = hg * kHeadsPerCta + hl;
      out[(((size_t)b * g.H + h) * (size_t)(a.nbt * per_t) + blk) * D + d] =
          pool_s[(which * kHeadsPerCta + hl) * D + d] * inv;
    }
  }
}

size_t prologue_smem_bytes(const Geo& g, int dt, int dh, int dw) {
  return (size_t)2 * kHeadsPerCta * g.D * sizeof(float) +
         (size_t)(g.bt * (dt / 2) + g.bh * (dh / 2) + g.bw * (dw / 2)) * sizeof(float2);
}

cudaError_t launch_prologue(const PrologueArgs& a, cudaStream_t s) {
  const Geo& g = a.g;
  dim3 grid(a.nbt * g.nbh * g.nbw, (g.H + kHeadsPerCta - 1) / kHeadsPerCta, g.B);
  size_t smem = prologue_smem_bytes(g, a.dt, a.dh, a.dw);
  const bool plain = a.sh.n == 1 && a.sh.h_stride == g.H && a.sh.h0 == 0;
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kPrologueThreads, smem, s>>>(a);
  };
  if (g.D == 128) plain ? go(prologue_kernel<128, false>) : go(prologue_kernel<128, true>);
  else plain ? go(prologue_kernel<64, false>) : go(prologue_kernel<64, true>);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------ backward
// Gradients of the prologue: dz (blocked, bf16) -> dx (raster, bf16) and, for q and k with a
// gain, dgamma.  Per (token, head) row, undoing the forward in reverse order:
//   RoPE:    dy = R(a)^T dz per pair (turned back by the forward angle);
//   RMSNorm: xh = x / r, r = sqrt(mean(x^2) + eps); dgamma += dy * xh;
//            dxh = dy * gamma; dx = (dxh - xh * mean(dxh * xh)) / r.
// v (and q / k without a gain and RoPE) is the inverse relayout.  Same tiling as the forward
// (one CTA per block of the padded grid and 8 heads); each thread keeps the dgamma partials
// of its 8 columns over its rows, the CTA sums them in shared memory and writes one partial
// row per CTA, and prologue_dgamma_kernel adds the partial rows in a fixed order, so dgamma
// is deterministic.
struct PrologueBwdArgs {
  PrologueArgs f;                 // geometry, RoPE widths, frames, t_offset, gamma, eps, theta
  const __nv_bfloat16* dz[3];     // blocked gradients of the outputs (NULL = skip)
  const __nv_bfloat16* x[2][kMaxShards];  // raster forward inputs q, k per shard (with a gain)
  __nv_bfloat16* dx[3][kMaxShards];       // raster gradients of the inputs per shard (f.sh)
  float* part[2];                 // [n_cta][D] dgamma partials of q, k
};

template <int D, bool kSharded>
__global__ void __launch_bounds__(kPrologueThreads)
    prologue_bwd_kernel(const PrologueBwdArgs a) {
  constexpr int LPR = D / 8;                     // lanes per row
  constexpr int RPP = kPrologueThreads / LPR;    // rows per pass
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float* gsum = reinterpret_cast<float*>(smem_raw);            // [2][D]
  float2* tab = reinterpret_cast<float2*>(gsum + 2 * D);

  const PrologueArgs& f = a.f;
  const Geo& g = f.g;
  const int blk = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x;
  const int per_t = g.nbh * g.nbw;
  const int ibt = blk / per_t, ibh = (blk % per_t) / g.nbw, ibw = blk % g.nbw;
  int vt, vh, vw;
  block_extent(g, f.frames, blk, vt, vh, vw);
  const int nvalid = max(vt, 0) * max(vh, 0) * max(vw, 0);
  const bool full = vh == g.bh && vw == g.bw;  // slot decode by shifts
  const bool rope = f.theta > 0.f;
  const int pt = f.dt / 2, ph = f.dh / 2;
  const int off_h = g.bt * pt, off_w = off_h + g.bh * ph;
  if (rope) build_rope_table(f, ibt, ibh, ibw, tab);
  for (int e = tid; e < 2 * D; e += kPrologueThreads) gsum[e] = 0.f;
  __syncthreads();

  const int rid = tid / LPR, cl = tid % LPR, c0 = cl * 8;
  const int heads_here = min(kHeadsPerCta, g.H - hg * kHeadsPerCta);
  const int hpc = kSharded ? heads_here : kHeadsPerCta;  // as in the forward
  const int rows = hpc * g.BS;
  const size_t n_raster = (size_t)f.frames * g.GH * g.GW;
  int ax[4], pi[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int pp = c0 / 2 + q;
    if (2 * pp < f.dt) { ax[q] = 0; pi[q] = pp; }
    else if (2 * pp < f.dt + f.dh) { ax[q] = 1; pi[q] = pp - pt; }
    else { ax[q] = 2; pi[q] = pp - pt - ph; }
  }
  for (int which = 0; which < 3; ++which) {
    const __nv_bfloat16* __restrict__ dz = a.dz[which];
    if (dz == nullptr) continue;
    const bool qk = which < 2;
    const float* gam = qk ? f.gamma[which] : nullptr;
    const bool do_rope = qk && rope;
    // the one shard of a plain call
    const __nv_bfloat16* __restrict__ xin0 = qk ? a.x[which][0] : nullptr;
    __nv_bfloat16* __restrict__ dx0 = a.dx[which][0];
    float gv[8], gacc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { gv[e] = gam ? gam[c0 + e] : 1.f; gacc[e] = 0.f; }
    for (int base = 0; base < rows; base += RPP) {
      const int row = base + rid;
      const int hl = row % hpc, slot = row / hpc;
      const int h = hg * kHeadsPerCta + hl;
      const bool valid = row < rows && hl < heads_here && slot < nvalid;
      int lt = 0, lh = 0, lw = 0;
      if (valid) slot_local(g, slot, vh, vw, full, lt, lh, lw);
      float v[8], xv[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) { v[e] = 0.f; xv[e] = 0.f; }
      size_t xoff = 0;
      int sidx = 0;
      if (valid) {
        const int t = ibt * g.bt + lt, hh = ibh * g.bh + lh, ww = ibw * g.bw + lw;
        xoff = shard_elem<kSharded, D>(f.sh, g, n_raster, b, t, hh, ww, h, c0, sidx);
        const uint4 rz = __ldg(reinterpret_cast<const uint4*>(
            dz + ((((size_t)b * g.H + h) * (size_t)(f.nbt * per_t) + blk) * g.BS + slot) * D + c0));
        const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&rz);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 ff = __bfloat1622float2(p2[e]);
          v[2 * e] = ff.x; v[2 * e + 1] = ff.y;
        }
        if (gam) {
          const uint4 rx = __ldg(reinterpret_cast<const uint4*>((kSharded ? a.x[which][sidx] : xin0) + xoff));
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&rx);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 ff = __bfloat1622float2(x2[e]);
            xv[2 * e] = ff.x; xv[2 * e + 1] = ff.y;
          }
        }
      }
      if (do_rope && valid) {  // dy = R(a)^T dz
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float2 cs;
          if (ax[q] == 0) cs = tab[lt * pt + pi[q]];
          else if (ax[q] == 1) cs = tab[off_h + lh * ph + pi[q]];
          else cs = tab[off_w + lw * (f.dw / 2) + pi[q]];
          const float z0 = v[2 * q], z1 = v[2 * q + 1];
          v[2 * q] = z0 * cs.x + z1 * cs.y;
          v[2 * q + 1] = -z0 * cs.y + z1 * cs.x;
        }
      }
      if (gam) {  // RMSNorm backward; every lane takes part in the shuffles
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(xv[e], xv[e], ss);
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rs = rsqrtf(ss * (1.0f / D) + f.eps);  // 1 / r
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float xh = xv[e] * rs;
          gacc[e] = fmaf(v[e], xh, gacc[e]);   // dgamma (pad rows add 0)
          v[e] *= gv[e];                        // d xh
          dot = fmaf(v[e], xh, dot);
        }
#pragma unroll
        for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        const float mdot = dot * (1.0f / D);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = (v[e] - xv[e] * rs * mdot) * rs;
      }
      if (valid) {
        uint4 outv;
        uint32_t* o32 = reinterpret_cast<uint32_t*>(&outv);
#pragma unroll
        for (int e = 0; e < 4; ++e) o32[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        *reinterpret_cast<uint4*>((kSharded ? a.dx[which][sidx] : dx0) + xoff) = outv;
      }
    }
    if (gam && a.part[which] != nullptr) {
#pragma unroll
      for (int e = 0; e < 8; ++e) atomicAdd(&gsum[which * D + c0 + e], gacc[e]);
    }
  }
  __syncthreads();
  const size_t cta = ((size_t)b * gridDim.y + hg) * gridDim.x + blk;
  for (int which = 0; which < 2; ++which) {
    if (a.part[which] == nullptr || a.dz[which] == nullptr || f.gamma[which] == nullptr) continue;
    for (int e = tid; e < D; e += kPrologueThreads) a.part[which][cta * D + e] = gsum[which * D + e];
  }
}

// dgamma[d] = sum over the CTAs' partial rows, in CTA order (deterministic).
__global__ void __launch_bounds__(256) prologue_dgamma_kernel(const float* __restrict__ part,
                                                              int n_cta, int d, float* __restrict__ out) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= d) return;
  float s = 0.f;
  for (int c = 0; c < n_cta; ++c) s += part[(size_t)c * d + e];
  out[e] = s;
}

int prologue_bwd_ctas(const Geo& g, int nbt) {
  return nbt * g.nbh * g.nbw * ((g.H + kHeadsPerCta - 1) / kHeadsPerCta) * g.B;
}

cudaError_t launch_prologue_bwd(const PrologueBwdArgs& a, float* dgamma[2], cudaStream_t s) {
  const Geo& g = a.f.g;
  dim3 grid(a.f.nbt * g.nbh * g.nbw, (g.H + kHeadsPerCta - 1) / kHeadsPerCta, g.B);
  const size_t smem = (size_t)2 * g.D * sizeof(float) +
                      (size_t)(g.bt * (a.f.dt / 2) + g.bh * (a.f.dh / 2) + g.bw * (a.f.dw / 2)) * sizeof(float2);
  const bool plain = a.f.sh.n == 1 && a.f.sh.h_stride == g.H && a.f.sh.h0 == 0;
  auto go = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    kern<<<grid, kPrologueThreads, smem, s>>>(a);
  };
  if (g.D == 128) plain ? go(prologue_bwd_kernel<128, false>) : go(prologue_bwd_kernel<128, true>);
  else plain ? go(prologue_bwd_kernel<64, false>) : go(prologue_bwd_kernel<64, true>);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_cta = (int)(grid.x * grid.y * grid.z);
  for (int w = 0; w < 2; ++w) {
    if (dgamma[w] == nullptr || a.part[w] == nullptr) continue;
    prologue_dgamma_kernel<<<(g.D + 255) / 256, 256, 0, s>>>(a.part[w], n_cta, g.D, dgamma[w]);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace bsa
