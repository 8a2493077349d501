// attn_fwd.cu -- sparse flash-attention forward over the selected key blocks (sm_100a).
//
// Source: "LongCat-Video视频生成模型发布 迈出世界模型探索第一步", section 块稀疏注意力（BSA）
// (attention is computed only over the top-r key blocks of each query block) and
// "LongCat-Video : Generate 1 minute long AI videos with this model", section "Sparse
// attention".  The pages' kernel rides on FlashAttention for older GPUs; this one is a
// Blackwell design: TMA tiles -> tcgen05.mma with accumulators in TMEM.
//
// Work item = (b, h, query block i): a 128-row Q tile (the block's BS slots first) against
// the K/V tiles of idx[b,h,i,0:cnt].  Persistent CTAs (one per SM), items in head-major
// order so the CTAs running at once share one head's K/V in L2.  Each CTA keeps two items
// in flight ("lanes" A and B) so one lane's softmax overlaps the other lane's MMAs.
//
// Warp roles (640 threads = 5 warpgroups):
//   warps 0-7   softmax + epilogue of lane A: warps 0-3 take the left half of every S row
//               (keys 0..BS/2-1), warps 4-7 the right half; thread = query row = TMEM lane
//   warps 8-15  the same for lane B
//   warp 16     TMA producer (one thread)
//   warp 17     MMA issuer (one thread); owns the TMEM allocation (512 columns)
//   warps 18-19 idle
// The two threads of a row exchange their partial row maxima through shared memory behind a
// named barrier of the lane's 256 threads, so both apply the same running max; each keeps a
// partial row sum, combined once per item.  Registers: launched at 96 per thread
// (640 x 96 = 61440); the control warpgroup drops to kRegsCtl and the softmax warpgroups
// rise to kRegsSoftmax: 512 * 104 + 128 * 56 = 60416 <= 61440.
// TMEM columns: lane L uses S/P at [256L, 256L+BS) and O at [256L+128, 256L+128+D).
// P (bf16) overwrites the first BS/2 columns of S; the next S of that lane is issued after
// the PV that reads P, and tcgen05 MMAs of one thread execute in issue order.
//
// Shared memory: Q tile per lane + a ring of kStages K/V tiles, consumed strictly in the
// order the MMA thread uses them; the producer walks the identical schedule.
// Online softmax in the exp2 domain with lazy rescaling: the running max is only raised
// when a row's max grows by more than 8 (log2 units), so O is rarely touched; the final
// O / l and LSE are exact either way.
#include "common.cuh"

namespace bsa {

struct FwdParams {
  Geo g;
  int r;
  int n_items;
  const int* idx;
  const int* cnt;
  __nv_bfloat16* o;
  float* lse;
};

constexpr int kFwdThreads = 640;
constexpr int kProducerWarp = 16, kMmaWarp = 17;
constexpr int kRegsLaunch = 96;  // 65536 / 640 rounded down to a multiple of 8
constexpr int kRegsSoftmax = 104;
constexpr int kRegsCtl = 56;
static_assert(512 * kRegsSoftmax + 128 * kRegsCtl <= kFwdThreads * kRegsLaunch,
              "register re-split exceeds the launch allocation");
constexpr int kFwdStages = 4;
constexpr int kTileM = 128;
// softmax arithmetic options (see the design doc for the measurements behind the defaults)
constexpr bool kPolyExp = false;   // half of the exponentials on the FMA pipe
constexpr bool kMax3 = true;       // 3-input max for the row max
constexpr bool kPacked = true;     // f32x2 FMA / ADD for the exponent argument and row sum

template <int BS, int D>
struct FwdLayout {
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = BS * D * 2;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = 2 * kQBytes;
  static constexpr int kBarOff = kRingOff + kFwdStages * kKVBytes;
  // barriers: q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] fin
  static constexpr int kNumBars = 2 * 5 + 2 * kFwdStages + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kXchOff = kMiscOff + 16;              // float [2 lanes][2 halves][128]
  static constexpr int kSumOff = kXchOff + 2 * 2 * 128 * 4;  // float [2 lanes][2 halves][128]
  static constexpr int kBytes = kSumOff + 2 * 2 * 128 * 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

// Cursor over the items of one lane: items blockIdx.x + gridDim.x * (2k + lane), skipping
// items with cnt == 0.  The producer and the MMA thread walk identical cursors.
struct Cursor {
  int k, item, cnt, n;
};

__device__ __forceinline__ int load_cnt(const FwdParams& p, int item) {
  int c = __ldg(p.cnt + item);
  if (c < 0 || c > p.r) {
    set_status(DEV_BAD_INDEX);
    c = c < 0 ? 0 : p.r;
  }
  return c;
}

__device__ __forceinline__ int load_idx(const FwdParams& p, int item, int n) {
  int j = __ldg(p.idx + (size_t)item * p.r + n);
  if (j < 0 || j >= p.g.NBk) {
    set_status(DEV_BAD_INDEX);
    j = 0;
  }
  return j;
}

__device__ __forceinline__ bool cursor_seek(const FwdParams& p, Cursor& c, int lane) {
  for (;; ++c.k) {
    const int item = blockIdx.x + gridDim.x * (2 * c.k + lane);
    if (item >= p.n_items) { c.item = -1; return false; }
    const int n = load_cnt(p, item);
    if (n > 0) { c.item = item; c.cnt = n; c.n = 0; return true; }
  }
}
__device__ __forceinline__ bool cursor_next(const FwdParams& p, Cursor& c, int lane) {
  if (++c.n < c.cnt) return true;
  ++c.k;
  return cursor_seek(p, c, lane);
}

template <int BS, int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const FwdParams p) {
  using L = FwdLayout<BS, D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 2;
  uint64_t* kv_full = bars + 4;
  uint64_t* kv_empty = kv_full + kFwdStages;
  uint64_t* s_full = kv_empty + kFwdStages;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* fin_bar = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const Geo& g = p.g;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 256);
      mbar_init(&o_full[i], 1);
    }
    for (int s = 0; s < kFwdStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(fin_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_holder, 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // every role ends here: all TMEM traffic done, then warp 9 releases the columns
  auto teardown = [&]() {
    tc_fence_before();
    named_bar_sync(1, kFwdThreads);
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem_base, 512);
  };

  if (warp >= kProducerWarp) {
  regs_dec<kRegsCtl>();
  if (warp == kProducerWarp) {
    // ================================================================ TMA producer
    // Walks the same schedule as the MMA thread: for each lane in turn, the V tile of the
    // current step, then (after advancing) the Q tile of a new item and the next K tile.
    // All state lives in registers (the two lanes are unrolled statically).
    if (lane == 0) {
      Cursor c0{0, -1, 0, 0}, c1{0, -1, 0, 0};
      bool a0 = cursor_seek(p, c0, 0), a1 = cursor_seek(p, c1, 1);
      int seq = 0, ql0 = 0, ql1 = 0;
      bool ok = true;
      unsigned char* ring = smem + L::kRingOff;
      auto kv_tile = [&](const Cursor& c, bool is_v) -> bool {
        const int stage = seq % kFwdStages, round = seq / kFwdStages;
        if (round > 0 && !mbar_wait(&kv_empty[stage], (round - 1) & 1, abort_flag)) return false;
        const int j = load_idx(p, c.item, c.n);
        const int bhx = c.item / g.NBq;
        const CUtensorMap* map;
        int row;
        if (j < g.NBc) { map = is_v ? &tmVc : &tmKc; row = (bhx * g.NBc + j) * BS; }
        else { map = is_v ? &tmV : &tmK; row = (bhx * g.NBq + (j - g.NBc)) * BS; }
        unsigned char* dst = ring + stage * L::kKVBytes;
        mbar_expect_tx(&kv_full[stage], L::kKVBytes);
#pragma unroll
        for (int half = 0; half < D / 64; ++half)
          tma_load_2d(dst + half * BS * 128, map, half * 64, row, &kv_full[stage]);
        ++seq;
        return true;
      };
      auto q_tile = [&](const Cursor& c, int lw, int& ql) -> bool {
        if (ql > 0 && !mbar_wait(&q_empty[lw], (ql - 1) & 1, abort_flag)) return false;
        unsigned char* dst = smem + L::kQOff + lw * L::kQBytes;
        mbar_expect_tx(&q_full[lw], L::kQBytes);
#pragma unroll
        for (int half = 0; half < D / 64; ++half)
          tma_load_2d(dst + half * kTileM * 128, &tmQ, half * 64, c.item * BS, &q_full[lw]);
        ++ql;
        return true;
      };
      if (a0) ok = q_tile(c0, 0, ql0) && kv_tile(c0, false);
      if (ok && a1) ok = q_tile(c1, 1, ql1) && kv_tile(c1, false);
      while (ok && (a0 || a1)) {
        if (a0) {
          ok = kv_tile(c0, true);
          if (!ok) break;
          a0 = cursor_next(p, c0, 0);
          if (a0) ok = (c0.n > 0 || q_tile(c0, 0, ql0)) && kv_tile(c0, false);
          if (!ok) break;
        }
        if (a1) {
          ok = kv_tile(c1, true);
          if (!ok) break;
          a1 = cursor_next(p, c1, 1);
          if (a1) ok = (c1.n > 0 || q_tile(c1, 1, ql1)) && kv_tile(c1, false);
        }
      }
      // drain: every issued TMA load must land before the CTA may exit
      for (int st = 0; st < kFwdStages; ++st) {
        const int loads = seq / kFwdStages + (st < seq % kFwdStages ? 1 : 0);
        if (loads > 0) mbar_wait_drain(&kv_full[st], (loads - 1) & 1);
      }
      if (ql0 > 0) mbar_wait_drain(&q_full[0], (ql0 - 1) & 1);
      if (ql1 > 0) mbar_wait_drain(&q_full[1], (ql1 - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileM, BS, 0, 0);
      constexpr uint32_t idPV = idesc_bf16(kTileM, D, 0, 1);
      Cursor c0{0, -1, 0, 0}, c1{0, -1, 0, 0};
      bool a0 = cursor_seek(p, c0, 0), a1 = cursor_seek(p, c1, 1);
      int seq = 0, qc0 = 0, qc1 = 0, pc0 = 0, pc1 = 0;
      bool ok = true;
      // descriptor bases; per-MMA descriptors add (byte offset >> 4) to the start field
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
      const uint64_t dq1 = smem_desc_sw128(smem_u32(smem + L::kQOff + L::kQBytes), 16, 1024);
      const uint64_t dk = smem_desc_sw128(smem_u32(smem + L::kRingOff), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(smem + L::kRingOff), BS * 128, 1024);
      auto issue_S = [&](const Cursor& c, int lw, uint64_t dq, int& qc) -> bool {
        if (c.n == 0) {
          if (!mbar_wait(&q_full[lw], qc & 1, abort_flag)) return false;
          ++qc;
        }
        const int stage = seq % kFwdStages;
        if (!mbar_wait(&kv_full[stage], (seq / kFwdStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_s = tmem_base + lw * 256;
        const uint64_t kb = dk + (uint64_t)((stage * L::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = dq + (uint64_t)(((kk / 4) * (kTileM * 128) + (kk % 4) * 32) >> 4);
          const uint64_t bd = kb + (uint64_t)(((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4);
          mma_ss(d_s, ad, bd, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&kv_empty[stage]);
        mma_commit(&s_full[lw]);
        if (c.n == c.cnt - 1) mma_commit(&q_empty[lw]);
        ++seq;
        return true;
      };
      auto issue_PV = [&](const Cursor& c, int lw, int& pc) -> bool {
        if (!mbar_wait(&p_full[lw], pc & 1, abort_flag)) return false;
        ++pc;
        const int stage = seq % kFwdStages;
        if (!mbar_wait(&kv_full[stage], (seq / kFwdStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t d_o = tmem_base + lw * 256 + 128, a_p = tmem_base + lw * 256;
        const uint64_t vb = dv + (uint64_t)((stage * L::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          mma_ts(d_o, a_p + kk * 8, vb + (uint64_t)((kk * 2048) >> 4), idPV,
                 (c.n > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[stage]);
        if (c.n == c.cnt - 1) mma_commit(&o_full[lw]);
        ++seq;
        return true;
      };
      if (a0) ok = issue_S(c0, 0, dq0, qc0);
      if (ok && a1) ok = issue_S(c1, 1, dq1, qc1);
      while (ok && (a0 || a1)) {
        if (a0) {
          ok = issue_PV(c0, 0, pc0);
          if (!ok) break;
          a0 = cursor_next(p, c0, 0);
          if (a0) ok = issue_S(c0, 0, dq0, qc0);
          if (!ok) break;
        }
        if (a1) {
          ok = issue_PV(c1, 1, pc1);
          if (!ok) break;
          a1 = cursor_next(p, c1, 1);
          if (a1) ok = issue_S(c1, 1, dq1, qc1);
        }
      }
      // all MMAs issued by this thread must finish before TMEM is released
      mma_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0);
    }
  }
  teardown();
  } else {
    regs_inc<kRegsSoftmax>();
    // ================================================================ softmax + epilogue
    constexpr int HC = BS / 2;  // S columns (keys) per thread
    constexpr int HO = D / 2;   // O columns per thread
    const int Lw = warp / 8, hf = (warp / 4) & 1, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    const uint32_t t_s = tmem_base + t_lane + Lw * 256;   // S / P of this lane
    const uint32_t t_sh = t_s + hf * HC;                  // this thread's S columns
    const uint32_t t_ph = t_s + hf * (HC / 2);            // this thread's P columns (bf16 pairs)
    const uint32_t t_oh = t_s + 128 + hf * HO;            // this thread's O columns
    float* xch = reinterpret_cast<float*>(smem + L::kXchOff) + Lw * 256;
    float* xsum = reinterpret_cast<float*>(smem + L::kSumOff) + Lw * 256;
    const int bar_id = 2 + Lw;
    const float sl2 = g.scale * 1.4426950408889634f;
    int scons = 0, ocons = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = blockIdx.x + gridDim.x * (2 * k + Lw);
      if (item >= p.n_items) break;
      const int cnt = load_cnt(p, item);
      const int i = item % g.NBq;
      // this row's query slot (rows >= BS belong to the tile's padding and are discarded)
      bool qvalid = false;
      if (row < BS) {
        int vt, vh, vw;
        block_extent(g, g.T, i, vt, vh, vw);
        const int lt = row / (g.bh * g.bw), lh = (row / g.bw) % g.bh, lw = row % g.bw;
        qvalid = lt < vt && lh < vh && lw < vw;
      }
      float m = -INFINITY, l = 0.f;
      for (int n = 0; n < cnt; ++n) {
        bool w_ok = mbar_wait(&s_full[Lw], scons & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        ++scons;
        tc_fence_after();
        const int j = load_idx(p, item, n);
        float s[HC];
        {
          uint32_t* sr = reinterpret_cast<uint32_t*>(s);
          if constexpr (HC == 64) tmem_ld64_wait(t_sh, sr);
          else tmem_ld16_wait(t_sh, sr);
        }
        // pad keys of a partial block get -inf (mask built without divisions per column)
        int vt, vh, vw;
        if (j < g.NBc) block_extent(g, g.Tc, j, vt, vh, vw);
        else block_extent(g, g.T, j - g.NBc, vt, vh, vw);
        if (vt < g.bt || vh < g.bh || vw < g.bw) {
          uint32_t vm[BS / 32];
          block_valid_mask<BS>(g, vt, vh, vw, vm);
#pragma unroll
          for (int c = 0; c < HC; ++c) {
            const int kc = hf * HC + c;
            if (!((vm[kc >> 5] >> (kc & 31)) & 1u)) s[c] = -INFINITY;
          }
        }
        float mx;
        {
          float a0 = s[0], a1 = s[1], a2 = s[2], a3 = s[3];
#pragma unroll
          for (int c = 4; c + 8 <= HC; c += 8) {
            a0 = max3f(a0, s[c], s[c + 1]);
            a1 = max3f(a1, s[c + 2], s[c + 3]);
            a2 = max3f(a2, s[c + 4], s[c + 5]);
            a3 = max3f(a3, s[c + 6], s[c + 7]);
          }
          mx = max3f(max3f(a0, a1, a2), a3,
                     fmaxf(s[HC - 4], fmaxf(s[HC - 3], fmaxf(s[HC - 2], s[HC - 1]))));
        }
        // exchange the half-row maxima (the partner's S columns are read by now, so the P
        // stores below may overwrite them)
        xch[hf * 128 + row] = mx;
        named_bar_sync(bar_id, 256);
        mx = fmaxf(mx, xch[(1 - hf) * 128 + row]) * sl2;
        // lazy rescale: a row raises its running max only when it grew by more than 8
        // (log2 units); both threads of a row take the same decision.  tcgen05.ld/st are
        // warp-collective, so a warp rescales together (alpha = 1 for rows that keep their
        // max).  The PV of step n-1 has completed: the S of step n was issued after it.
        const float m_new = (n == 0 || mx > m + 8.0f) ? mx : m;
        const bool resc = n > 0 && m_new != m;
        if (__any_sync(0xffffffffu, resc)) {
          const float alpha = resc ? fast_exp2(m - m_new) : 1.0f;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < HO / 32; ++c) {
            uint32_t r32[32];
            tmem_ld32_wait(t_oh + c * 32, r32);
#pragma unroll
            for (int e = 0; e < 32; ++e) r32[e] = __float_as_uint(__uint_as_float(r32[e]) * alpha);
            tmem_st32(t_oh + c * 32, r32);
          }
          tmem_wait_st();
        }
        m = m_new;
        // P = exp2(s * scale * log2e - m) as bf16 pairs into this half's P columns
        const uint64_t sl2x2 = f2pack(sl2, sl2), nmx2 = f2pack(-m, -m);
        uint64_t sum2 = f2pack(0.f, 0.f);
#pragma unroll
        for (int c = 0; c < HC / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2unpack(fma2(f2pack(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]), sl2x2, nmx2), x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            sum2 = add2(sum2, f2pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_ph + c * 16, pk);
        }
        if constexpr (HC % 32 != 0) {  // BS = 32: 16 keys per thread, 8 P columns
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float x0, x1;
            f2unpack(fma2(f2pack(s[2 * e], s[2 * e + 1]), sl2x2, nmx2), x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            sum2 = add2(sum2, f2pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st8(t_ph, pk);
        }
        {
          float l0, l1;
          f2unpack(sum2, l0, l1);
          l += l0 + l1;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[Lw]);
      }
      if (!ok) break;
      float* lse_row = p.lse + (size_t)item * BS;
      __nv_bfloat16* o_row = p.o + ((size_t)item * BS + row) * D + hf * HO;
      if (cnt == 0) {
        if (row < BS) {
          uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < HO / 8; ++c) reinterpret_cast<uint4*>(o_row)[c] = z;
          if (hf == 0) lse_row[row] = -INFINITY;
        }
        continue;
      }
      // combine the two partial row sums (own buffer: the max exchange may already be in
      // use for the next item)
      xsum[hf * 128 + row] = l;
      named_bar_sync(bar_id, 256);
      l += xsum[(1 - hf) * 128 + row];
      bool w_ok = mbar_wait(&o_full[Lw], ocons & 1, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) { ok = false; break; }
      ++ocons;
      tc_fence_after();
      const float inv_l = qvalid ? 1.0f / l : 0.f;
#pragma unroll
      for (int c = 0; c < HO / 32; ++c) {
        uint32_t r32[32];
        tmem_ld32_wait(t_oh + c * 32, r32);
        if (row < BS) {
          uint4 v[4];
          uint32_t* v32 = reinterpret_cast<uint32_t*>(v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v32[e] = pack_bf16x2(__uint_as_float(r32[2 * e]) * inv_l,
                                 __uint_as_float(r32[2 * e + 1]) * inv_l);
#pragma unroll
          for (int e = 0; e < 4; ++e) reinterpret_cast<uint4*>(o_row + c * 32)[e] = v[e];
        }
      }
      if (row < BS && hf == 0)
        lse_row[row] = qvalid ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
      // the partner must have read this thread's partial sum before it is overwritten by
      // the next item's: the next write happens after the next item's first exchange
      // barrier, which the partner reaches only after reading it.
    }
    teardown();
  }
}

cudaError_t launch_fwd(const CUtensorMap* maps, const FwdParams& p, int n_sm, cudaStream_t s) {
  const int bs = p.g.BS, d = p.g.D;
  int grid = min(n_sm, (p.n_items + 1) / 2);
  if (grid < 1) grid = 1;
#define BSA_LAUNCH_FWD(BSv, Dv)                                                                    \
  do {                                                                                             \
    auto kern = bsa_fwd_kernel<BSv, Dv>;                                                           \
    const int smem = FwdLayout<BSv, Dv>::kAlloc;                                                   \
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); \
    if (e != cudaSuccess) return e;                                                                \
    kern<<<grid, kFwdThreads, smem, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);         \
    return cudaGetLastError();                                                                     \
  } while (0)
  if (bs == 128 && d == 128) BSA_LAUNCH_FWD(128, 128);
  if (bs == 128 && d == 64) BSA_LAUNCH_FWD(128, 64);
  if (bs == 32 && d == 128) BSA_LAUNCH_FWD(32, 128);
  if (bs == 32 && d == 64) BSA_LAUNCH_FWD(32, 64);
#undef BSA_LAUNCH_FWD
  return cudaErrorInvalidValue;
}

}  // namespace bsa
