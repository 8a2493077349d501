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
// order so the CTAs running at once share one head's K/V in L2.
//
// Two items per CTA in ping-pong: slot 0 takes the CTA's even-numbered items, slot 1 its
// odd ones, and the single MMA thread alternates between them, so the tensor cores compute
// one slot's S and P.V while the other slot's softmax runs.  Per slot: S = Q K^T into its own
// 128 TMEM columns (P, bf16, is written back over them), O in another 128; both slots fill
// the 512 columns.  S reads Q and K from shared memory (Q stays staged for the whole item).
//
// Warp roles (320 threads, so a thread may hold up to ~200 registers):
//   warps 0-3  slot 0 softmax + epilogue, warps 4-7 slot 1: warp w owns query rows
//              32*(w%4)..+31 (its TMEM lane quarter) and a thread owns a whole row, so the
//              row max needs no exchange between threads
//   warp 8     TMA producer (one thread): K / V tiles in the MMA thread's order
//   warp 9     MMA issuer (one thread); owns the TMEM allocation
// MMA order (per slot): S(0) | PV(0), S(1) | PV(1), S(2) | ... | PV(cnt-1), alternating
// slots group by group.  S(n+1) is written over P(n) after PV(n) has read it (tcgen05 MMAs
// of one thread run in issue order).  A slot's S-ready commit follows its previous PV in
// issue order, so when the softmax sees S(n) complete, O already holds P(0..n-1) V: the lazy
// rescale of O needs no further wait.  The softmax warps of a slot load the slot's next Q as
// soon as the current item's last S is complete (its last reader).
//
// Online softmax in the exp2 domain with lazy rescaling: the running max is raised only when
// a row's max grows by more than 8 (log2 units), so O is rarely touched; the final O / l and
// LSE are exact either way.
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

constexpr int kFwdThreads = 320;
constexpr int kSlotThreads = 128;  // softmax threads of one slot
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kFwdStages = 5;
constexpr int kTileM = 128;

template <int BS, int D>
struct FwdLayout {
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = BS * D * 2;
  static constexpr int kQOff = 0;                       // Q of slot s at kQOff + s * kQBytes
  static constexpr int kRingOff = 2 * kQBytes;
  static constexpr int kBarOff = kRingOff + kFwdStages * kKVBytes;
  // q_full[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] fin
  static constexpr int kNumBars = 2 + 2 * kFwdStages + 2 + 2 + 2 + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kMiscOff + 16;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
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

// The k-th item of slot s of this CTA: items blockIdx.x + (2k + s) * gridDim.x.
__device__ __forceinline__ int slot_item(int s, int k) {
  return (int)blockIdx.x + (2 * k + s) * (int)gridDim.x;
}

template <int BS, int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const FwdParams p) {
  using L = FwdLayout<BS, D>;
  constexpr int S = kFwdStages;
  static_assert(BS <= 128 && D <= 128, "one slot's S and O fit 128 TMEM columns each");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;            // [2] Q of the slot's next item staged (TMA)
  uint64_t* kv_full = bars + 2;       // [S]
  uint64_t* kv_empty = kv_full + S;   // [S]
  uint64_t* s_full = kv_empty + S;    // [2] S(n) of the slot in TMEM
  uint64_t* p_full = s_full + 2;      // [2] P(n) of the slot in TMEM (kSlotThreads arrivals)
  uint64_t* o_full = p_full + 2;      // [2] O of the slot's item complete
  uint64_t* fin_bar = o_full + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const Geo& g = p.g;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], kSlotThreads);
      mbar_init(&o_full[s], 1);
    }
    for (int s = 0; s < S; ++s) {
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
  // TMEM columns of slot s: S at 256 s, O at 256 s + 128
  auto t_s_col = [&](int s) -> uint32_t { return tmem_base + 256u * s; };
  auto t_o_col = [&](int s) -> uint32_t { return tmem_base + 256u * s + 128u; };
  // next item of slot s with a non-empty selection, from its k-th item on (k advanced)
  auto next_slot_item = [&](int s, int& k, int& cnt) -> int {
    for (;;) {
      const int it = slot_item(s, k);
      if (it >= p.n_items) return -1;
      cnt = load_cnt(p, it);
      if (cnt > 0) return it;
      ++k;
    }
  };

  if (warp == kProducerWarp) {
    // ================================================================ TMA producer
    // Walks the MMA thread's turn sequence (slot 0, slot 1, slot 0, ... skipping a finished
    // slot): a slot's first turn of an item loads K(0); its turn n loads V(n) and, unless n is
    // the item's last step, K(n+1).  Key-block indices are loaded a step ahead.
    if (lane == 0) {
      int seq = 0;
      bool ok = true;
      unsigned char* ring = smem + L::kRingOff;
      auto kv_tile = [&](int bhx, int j, bool is_v) -> bool {
        const int stage = seq % S, round = seq / S;
        if (round > 0 && !mbar_wait(&kv_empty[stage], (round - 1) & 1, abort_flag)) return false;
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
      // the two slots' states in registers: `a` takes this turn, then the two swap when the
      // other slot still has work (the turn order the MMA thread follows too)
      struct Slot { int s, k, item, cnt, n, jcur, jnext; };  // jcur / jnext: blocks of V(n), K(n+1)
      Slot a{0, 0, -1, 0, -1, 0, 0}, b{1, 0, -1, 0, -1, 0, 0};
      a.item = next_slot_item(0, a.k, a.cnt);
      b.item = next_slot_item(1, b.k, b.cnt);
      while (ok && (a.item >= 0 || b.item >= 0)) {
        if (a.item < 0) { const Slot t = a; a = b; b = t; }
        const int it = a.item, bhx = it / g.NBq;
        if (a.n < 0) {  // first turn of the item: K(0)
          a.jcur = load_idx(p, it, 0);
          a.jnext = a.cnt > 1 ? load_idx(p, it, 1) : 0;
          ok = kv_tile(bhx, a.jcur, false);
          a.n = 0;
        } else {  // turn n: V(n), then K(n+1)
          const int nn = a.n;
          const int jn2 = nn + 2 < a.cnt ? load_idx(p, it, nn + 2) : 0;  // a step ahead
          ok = kv_tile(bhx, a.jcur, true);
          if (ok && nn + 1 < a.cnt) ok = kv_tile(bhx, a.jnext, false);
          a.jcur = a.jnext;
          a.jnext = jn2;
          if (nn + 1 < a.cnt) {
            a.n = nn + 1;
          } else {  // item done: the slot's next item
            ++a.k;
            a.item = next_slot_item(a.s, a.k, a.cnt);
            a.n = -1;
          }
        }
        if (b.item >= 0) { const Slot t = a; a = b; b = t; }
      }
      // drain: every issued TMA load must land before the CTA may exit
      for (int st = 0; st < S; ++st) {
        const int loads = seq / S + (st < seq % S ? 1 : 0);
        if (loads > 0) mbar_wait_drain(&kv_full[st], (loads - 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileM, BS, 0, 0);
      constexpr uint32_t idPV = idesc_bf16(kTileM, D, 0, 1);
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(smem + L::kRingOff), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(smem + L::kRingOff), BS * 128, 1024);
      int seq = 0;
      bool ok = true;
      auto wait_tile = [&]() -> int {
        const int stage = seq % S;
        if (!mbar_wait(&kv_full[stage], (seq / S) & 1, abort_flag)) return -1;
        ++seq;
        return stage;
      };
      // S of slot s = Q_s K^T: A = Q (128 rows, K-major), B = the K tile in `stage`
      auto mma_S = [&](int s, int stage) {
        const uint64_t qd = dq0 + (uint64_t)((s * L::kQBytes) >> 4);
        const uint64_t kd = dk0 + (uint64_t)((stage * L::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = ((kk / 4) * (kTileM * 128) + (kk % 4) * 32) >> 4;
          const uint32_t offk = ((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4;
          mma_ss(t_s_col(s), qd + offq, kd + offk, idS, kk > 0 ? 1u : 0u);
        }
      };
      // the two slots' states in registers, swapped after each turn as in the producer
      struct Slot { int s, k, item, cnt, n, qc, pc; };  // qc / pc: Q loads, P(n) consumed
      Slot a{0, 0, -1, 0, -1, 0, 0}, b{1, 0, -1, 0, -1, 0, 0};
      a.item = next_slot_item(0, a.k, a.cnt);
      b.item = next_slot_item(1, b.k, b.cnt);
      while (ok && (a.item >= 0 || b.item >= 0)) {
        if (a.item < 0) { const Slot t = a; a = b; b = t; }
        const int s = a.s;
        if (a.n < 0) {  // S(0) once the slot's Q has landed
          const int sk = wait_tile();
          if (sk < 0 || !mbar_wait(&q_full[s], a.qc & 1, abort_flag)) { ok = false; break; }
          ++a.qc;
          tc_fence_after();
          mma_S(s, sk);
          mma_commit(&s_full[s]);
          mma_commit(&kv_empty[sk]);
          a.n = 0;
        } else {
          // turn n: O += P(n) V(n) (A = P from TMEM), then S(n+1) over P(n)
          const int nn = a.n;
          const bool more = nn + 1 < a.cnt;
          const int sv = wait_tile();
          const int sk = (sv >= 0 && more) ? wait_tile() : -1;
          if (sv < 0 || (more && sk < 0)) { ok = false; break; }
          if (!mbar_wait(&p_full[s], a.pc & 1, abort_flag)) { ok = false; break; }
          ++a.pc;
          tc_fence_after();
          const uint64_t vd = dv0 + (uint64_t)((sv * L::kKVBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BS / 16; ++kk)
            mma_ts(t_o_col(s), t_s_col(s) + kk * 8, vd + (uint64_t)((kk * 2048) >> 4), idPV,
                   (nn > 0 || kk > 0) ? 1u : 0u);
          if (more) {
            mma_S(s, sk);
            mma_commit(&s_full[s]);
            mma_commit(&kv_empty[sk]);
            a.n = nn + 1;
          } else {
            mma_commit(&o_full[s]);
            ++a.k;
            a.item = next_slot_item(s, a.k, a.cnt);
            a.n = -1;
          }
          mma_commit(&kv_empty[sv]);
        }
        if (b.item >= 0) { const Slot t = a; a = b; b = t; }
      }
      // all MMAs issued by this thread must finish before TMEM is released
      mma_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0);
    }
  } else {
    // ================================================================ softmax + epilogue
    const int s = warp / 4, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    const uint32_t t_s = t_s_col(s) + t_lane, t_o = t_o_col(s) + t_lane;
    const float sl2 = g.scale * 1.4426950408889634f;
    const bool leader = quarter == 0 && lane == 0;  // issues the slot's Q loads
    unsigned char* qbuf = smem + L::kQOff + s * L::kQBytes;
    int qloads = 0, gs = 0, oc = 0;  // Q loads issued, S steps consumed, items finished
    bool ok = true;
    auto load_q = [&](int item) {
      mbar_expect_tx(&q_full[s], L::kQBytes);
#pragma unroll
      for (int half = 0; half < D / 64; ++half)
        tma_load_2d(qbuf + half * kTileM * 128, &tmQ, half * 64, item * BS, &q_full[s]);
    };
    {
      int k0 = 0, c0 = 0;
      const int first = next_slot_item(s, k0, c0);
      if (leader && first >= 0) { load_q(first); ++qloads; }
    }
    // items of this slot, empty ones included (their O rows are zeros, LSE -inf)
    for (int kk = 0; ok; ++kk) {
      const int it = slot_item(s, kk);
      if (it >= p.n_items) break;
      const int c = load_cnt(p, it);
      const int i = it % g.NBq;
      const bool qvalid = row < BS && row < query_block_nvalid(g, i);
      float* lse_row = p.lse + (size_t)it * BS;
      __nv_bfloat16* o_row = p.o + ((size_t)it * BS + row) * D;
      if (c == 0) {
        if (row < BS) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int e = 0; e < D / 8; ++e) reinterpret_cast<uint4*>(o_row)[e] = z;
          lse_row[row] = -INFINITY;
        }
        continue;
      }
      // the slot's next non-empty item (its Q is loaded once this item's last S is done)
      int kn = kk + 1, cn = 0;
      const int nxt = next_slot_item(s, kn, cn);
      float m = -INFINITY, l = 0.f;
      // key-block valid counts 32 steps at a time (lane e holds step n0 + e), the next chunk's
      // index load in flight
      int jnext = lane < c ? load_idx(p, it, lane) : 0;
      int nreg = BS;
      uint32_t partial = 0;
      for (int n = 0; n < c; ++n, ++gs) {
        if ((n & 31) == 0) {
          const int jcur = jnext;
          jnext = n + 32 + lane < c ? load_idx(p, it, n + 32 + lane) : 0;
          nreg = n + lane < c ? key_block_nvalid(g, jcur) : BS;
          partial = __ballot_sync(0xffffffffu, nreg < BS);
        }
        bool w_ok = mbar_wait(&s_full[s], gs & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
        // S(c-1) complete: Q of this item has no reader left; stage the next item's Q
        if (n == c - 1 && leader && nxt >= 0) { load_q(nxt); ++qloads; }
        // the row of S (BS fp32 values) in registers; pad keys of a partial block (its slots
        // >= its valid count) count as -inf
        float sv[BS];
        {
          uint32_t* sr = reinterpret_cast<uint32_t*>(sv);
          if constexpr (BS == 128) tmem_ld128_wait(t_s, sr);
          else tmem_ld32_wait(t_s, sr);
        }
        if ((partial >> (n & 31)) & 1u) {
          const int nv = __shfl_sync(0xffffffffu, nreg, n & 31);
#pragma unroll
          for (int e = 0; e < BS; ++e)
            if (e >= nv) sv[e] = -INFINITY;
        }
        float mx;
        {  // four independent max3 chains over the row (BS is a multiple of 8)
          float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
          for (int e = 0; e < BS; e += 8) {
            a0 = max3f(a0, sv[e], sv[e + 1]);
            a1 = max3f(a1, sv[e + 2], sv[e + 3]);
            a2 = max3f(a2, sv[e + 4], sv[e + 5]);
            a3 = max3f(a3, sv[e + 6], sv[e + 7]);
          }
          mx = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3)) * sl2;
        }
        // lazy rescale: raise the running max only when it grew by more than 8 (log2 units).
        // O holds P(0..n-1) V already (S(n)'s commit followed PV(n-1)); tcgen05.ld/st are
        // warp-collective, so a warp rescales together (alpha = 1 for rows that keep their max)
        const float m_new = (n == 0 || mx > m + 8.0f) ? mx : m;
        const bool resc = n > 0 && m_new != m;
        if (__any_sync(0xffffffffu, resc)) {
          const float alpha = resc ? fast_exp2(m - m_new) : 1.0f;
          l *= alpha;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            tmem_ld32_wait(t_o + c0, r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(t_o + c0, r);
          }
          tmem_wait_st();
        }
        m = m_new;
        // P = exp2(s * scale * log2e - m) as bf16 pairs over the first BS/2 columns of S
        const uint64_t sl2x2 = f2pack(sl2, sl2), nmx2 = f2pack(-m, -m);
        uint64_t sum2 = f2pack(0.f, 0.f);
#pragma unroll
        for (int c0 = 0; c0 < BS; c0 += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float x0, x1;
            f2unpack(fma2(f2pack(sv[c0 + 2 * e], sv[c0 + 2 * e + 1]), sl2x2, nmx2), x0, x1);
            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
            sum2 = add2(sum2, f2pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(t_s + c0 / 2, pk);
        }
        {
          float l0, l1;
          f2unpack(sum2, l0, l1);
          l += l0 + l1;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[s]);
      }
      if (!ok) break;
      // epilogue: O / l and LSE of this row, once the item's last PV has completed
      bool w_ok = mbar_wait(&o_full[s], oc & 1, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) { ok = false; break; }
      ++oc;
      tc_fence_after();
      const float inv_l = qvalid ? 1.0f / l : 0.f;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld32_wait(t_o + c0, r);
        if (row < BS) {
          uint4 v[4];
          uint32_t* v32 = reinterpret_cast<uint32_t*>(v);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v32[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
#pragma unroll
          for (int e = 0; e < 4; ++e) reinterpret_cast<uint4*>(o_row + c0)[e] = v[e];
        }
      }
      if (row < BS) lse_row[row] = qvalid ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
    }
    // every Q load this slot issued must land before the CTA may exit
    if (leader && qloads > 0) mbar_wait_drain(&q_full[s], (qloads - 1) & 1);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, 512);
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
