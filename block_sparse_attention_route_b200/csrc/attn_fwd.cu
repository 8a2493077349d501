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
// Warp roles (576 threads; 18 warps put 5 on two SM sub-partitions, so at most 96 registers):
//   warps 0-15  softmax + epilogue: warp w reads TMEM lanes 32*(w%4).. (query rows) and owns
//               the key-column group w/4 (BS/4 keys) of every S tile and the O-column group
//               w/4 (D/4 columns) of the output
//   warp 16     TMA producer (one thread)
//   warp 17     MMA issuer (one thread); owns the TMEM allocation
// TMEM columns: S0 [0,128), S1 [128,256), O [256,256+D), Q slots [256+D, 256+2D) (two of
// D/2 columns: bf16 pairs).  Q is the A operand of S = Q K^T straight from TMEM, so the
// tensor cores read only K from shared memory for S (a shared-memory-bandwidth saving: an SS
// MMA pair of 128x16 bf16 tiles reads 8 KB per 64 clocks, the whole 128 B/clock).  The
// softmax warps copy each item's Q from its staging tile into a Q slot one item ahead.
// S is double buffered: while the
// softmax turns S(n) into P(n) (bf16, written over the first BS/2 columns of its buffer),
// the tensor cores already compute S(n+1).  MMA order: S(0), S(1), then per step PV(n) and
// S(n+2) into the buffer P(n) came from (tcgen05 MMAs of one thread run in issue order, so
// S(n+2) is written after PV(n) has read P(n)).
//
// The four column groups of a row (warps q, q+4, q+8, q+12: the same TMEM lanes) exchange
// partial row maxima through shared memory behind a named barrier of those 128 threads (one
// per step; the exchange slots alternate with the step parity) and keep partial row sums,
// combined once per item.  The barrier also orders every group's read of S(n) before any
// group overwrites it with P(n).  The four row quarters run independently: P-ready is one
// mbarrier per S buffer, so the phases of one barrier are two steps apart and a quarter can
// never arrive for step n+2 before the MMA thread has consumed step n (S(n+2) is issued only
// after PV(n)).  Online softmax in the exp2 domain with lazy
// rescaling: the running max is raised only when a row's max grows by more than 8 (log2
// units), so O is rarely touched (and then only after the previous PV has completed, which
// the pv_done barrier tells); the final O / l and LSE are exact either way.
//
// Shared memory: two Q staging buffers and a ring of K/V tiles consumed strictly in the order
// the MMA thread uses them; the producer walks the identical schedule.  Q of the j-th
// non-empty item of a CTA is staged in buffer j & 1 and copied to TMEM slot j & 1: the
// producer loads Q(j+1) before the K/V tiles of item j, the softmax warps copy it during step
// 0 of item j (its slot's previous Q, item j-1's, is no longer read: every S of item j-1
// completed before S(0) of item j) and free the staging buffer, and the MMA thread waits for
// the copy before the first S of item j+1.
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

constexpr int kFwdThreads = 576;
constexpr int kSoftmaxThreads = 512;
constexpr int kProducerWarp = 16, kMmaWarp = 17;
constexpr int kFwdStages = 5;
constexpr int kQBufs = 1;  // Q staging buffers (Q leaves for TMEM at step 0 of the item before)
constexpr int kTileM = 128;

template <int BS, int D>
struct FwdLayout {
  static constexpr int kQBytes = kTileM * D * 2;
  static constexpr int kKVBytes = BS * D * 2;
  static constexpr int kQOff = 0;
  static constexpr int kRingOff = kQBufs * kQBytes;
  static constexpr int kBarOff = kRingOff + kFwdStages * kKVBytes;
  // q_full[2] q_empty[2] qt_full[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] pv_done o_full fin
  static constexpr int kNumBars = 6 + 2 * kFwdStages + 2 + 2 + 3;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kXchOff = kMiscOff + 16;               // float [2 parity][4 groups][128]
  static constexpr int kSumOff = kXchOff + 2 * 4 * 128 * 4;   // float [4 groups][128]
  static constexpr int kBytes = kSumOff + 4 * 128 * 4;
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

template <int BS, int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKc,
                   const __grid_constant__ CUtensorMap tmVc, const FwdParams p) {
  using L = FwdLayout<BS, D>;
  constexpr int S = kFwdStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;            // [2] Q staged (TMA)
  uint64_t* q_empty = bars + 2;       // [2] staging buffer copied out (kSoftmaxThreads arrivals)
  uint64_t* qt_full = bars + 4;       // [2] Q in its TMEM slot (kSoftmaxThreads arrivals)
  uint64_t* kv_full = bars + 6;       // [S]
  uint64_t* kv_empty = kv_full + S;   // [S]
  uint64_t* s_full = kv_empty + S;    // [2] S(n) in buffer n & 1
  uint64_t* p_full = s_full + 2;      // [2] P(n) written into buffer n & 1 (kSoftmaxThreads arrivals)
  uint64_t* pv_done = p_full + 2;     // PV(n) complete
  uint64_t* o_full = pv_done + 1;     // O of the item complete
  uint64_t* fin_bar = o_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const Geo& g = p.g;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], kSoftmaxThreads);
      mbar_init(&qt_full[i], kSoftmaxThreads);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], kSoftmaxThreads);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_full, 1);
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
  const uint32_t t_o0 = tmem_base + 256;
  const uint32_t t_q0 = tmem_base + 256 + D;  // Q slot b at t_q0 + b * D / 2
  // next item with a non-empty selection at or after `it` in this CTA's sequence
  auto next_item = [&](int it) {
    while (it < p.n_items && load_cnt(p, it) == 0) it += gridDim.x;
    return it;
  };

  if (warp == kProducerWarp) {
    // ================================================================ TMA producer
    // Load order = MMA consumption order: per item K(0), K(1), then per step n: V(n),
    // K(n+2); Q of the next non-empty item is staged before the current item's tiles.
    if (lane == 0) {
      int seq = 0, items = 0;
      bool ok = true;
      unsigned char* ring = smem + L::kRingOff;
      // K or V tile of key block j of head row bhx into the next ring stage
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
      // Q of the `items`-th non-empty item into staging buffer items % kQBufs (free once the
      // softmax warps copied out the Q kQBufs items back)
      auto q_tile = [&](int item) -> bool {
        const int qb = items % kQBufs;
        if (items >= kQBufs &&
            !mbar_wait(&q_empty[qb], ((items / kQBufs) - 1) & 1, abort_flag)) return false;
        mbar_expect_tx(&q_full[qb], L::kQBytes);
#pragma unroll
        for (int half = 0; half < D / 64; ++half)
          tma_load_2d(smem + L::kQOff + qb * L::kQBytes + half * kTileM * 128, &tmQ, half * 64,
                      item * BS, &q_full[qb]);
        ++items;
        return true;
      };
      int item = next_item(blockIdx.x);
      if (item < p.n_items) ok = q_tile(item);
      while (item < p.n_items && ok) {
        const int cnt = load_cnt(p, item);
        const int nxt = next_item(item + gridDim.x);
        if (nxt < p.n_items) ok = q_tile(nxt);
        // Key-block indices of steps n, n+1, n+2 ride in registers and the index of step n+3
        // is loaded one step ahead, so no global-load latency sits in the chain of waits and
        // TMA issues (each index is loaded once, for its K tile, and reused for its V tile).
        const int bhx = item / g.NBq;
        int j0 = load_idx(p, item, 0), j1 = cnt > 1 ? load_idx(p, item, 1) : 0;
        int j2 = cnt > 2 ? load_idx(p, item, 2) : 0;
        ok = ok && kv_tile(bhx, j0, false) && (cnt < 2 || kv_tile(bhx, j1, false));
        for (int n = 0; n < cnt && ok; ++n) {
          const int j3 = n + 3 < cnt ? load_idx(p, item, n + 3) : 0;  // used next step
          ok = kv_tile(bhx, j0, true);                                 // V(n)
          if (ok && n + 2 < cnt) ok = kv_tile(bhx, j2, false);         // K(n+2)
          j0 = j1; j1 = j2; j2 = j3;
        }
        item = nxt;
      }
      // drain: every issued TMA load must land before the CTA may exit
      for (int st = 0; st < S; ++st) {
        const int loads = seq / S + (st < seq % S ? 1 : 0);
        if (loads > 0) mbar_wait_drain(&kv_full[st], (loads - 1) & 1);
      }
      for (int b = 0; b < kQBufs; ++b) {
        const int loads = items / kQBufs + (b < items % kQBufs ? 1 : 0);
        if (loads > 0) mbar_wait_drain(&q_full[b], (loads - 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTileM, BS, 0, 0);
      constexpr uint32_t idPV = idesc_bf16(kTileM, D, 0, 1);
      const uint64_t dk = smem_desc_sw128(smem_u32(smem + L::kRingOff), 16, 1024);
      const uint64_t dv = smem_desc_sw128(smem_u32(smem + L::kRingOff), BS * 128, 1024);
      int seq = 0, items = 0, gs = 0, gp = 0;  // ring position, items, S issued, P consumed
      bool ok = true;
      auto wait_tile = [&]() -> int {
        const int stage = seq % S;
        if (!mbar_wait(&kv_full[stage], (seq / S) & 1, abort_flag)) return -1;
        tc_fence_after();
        return stage;
      };
      // S(gs) = Q K^T into buffer gs & 1: A = Q from TMEM slot a_q (K16 slice kk at column
      // 8 kk), B = the K tile in ring stage `stage`
      auto mma_S = [&](uint32_t a_q, int stage) {
        const uint64_t kb = dk + (uint64_t)((stage * L::kKVBytes) >> 4);
        const uint32_t d_s = tmem_base + (gs & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = ((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4;
          mma_ts(d_s, a_q + kk * 8, kb + offk, idS, kk > 0 ? 1u : 0u);
        }
      };
      // Every wait comes before the MMAs it guards, so each step issues one uninterrupted
      // group (PV(n) then S(n+2): 2 * D/16 or BS/16 + D/16 MMAs) followed by its commits;
      // a wait or commit between MMAs would let the tensor pipe drain.
      int cnt_next = (int)blockIdx.x < p.n_items ? load_cnt(p, blockIdx.x) : 0;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const int cnt = cnt_next;
        cnt_next = item + (int)gridDim.x < p.n_items ? load_cnt(p, item + gridDim.x) : 0;
        if (cnt == 0) continue;
        const int qb = items & 1;
        if (!mbar_wait(&qt_full[qb], (items >> 1) & 1, abort_flag)) { ok = false; break; }
        ++items;
        const int k0 = wait_tile();
        ++seq;
        const int k1 = (k0 >= 0 && cnt >= 2) ? wait_tile() : -1;
        if (cnt >= 2) ++seq;
        if (k0 < 0 || (cnt >= 2 && k1 < 0)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dq = t_q0 + qb * (D / 2);
        const int gs0 = gs;
        mma_S(dq, k0);
        ++gs;
        if (cnt >= 2) { mma_S(dq, k1); ++gs; }
        mma_commit(&s_full[gs0 & 1]);
        if (cnt >= 2) mma_commit(&s_full[(gs0 + 1) & 1]);
        mma_commit(&kv_empty[k0]);
        if (cnt >= 2) mma_commit(&kv_empty[k1]);
        for (int n = 0; n < cnt && ok; ++n) {
          const int sv = wait_tile();
          ++seq;
          const bool more = n + 2 < cnt;
          const int sk = (sv >= 0 && more) ? wait_tile() : -1;
          if (more) ++seq;
          if (sv < 0 || (more && sk < 0)) { ok = false; break; }
          // O += P(n) V(n): A = P from TMEM (buffer gp & 1), B = V (MN-major)
          if (!mbar_wait(&p_full[gp & 1], (gp >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t vb = dv + (uint64_t)((sv * L::kKVBytes) >> 4);
          const uint32_t a_p = tmem_base + (gp & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < BS / 16; ++kk)
            mma_ts(t_o0, a_p + kk * 8, vb + (uint64_t)((kk * 2048) >> 4), idPV,
                   (n > 0 || kk > 0) ? 1u : 0u);
          if (more) {  // S(n+2) into the buffer P(n) came from (read above, in issue order)
            mma_S(dq, sk);
            mma_commit(&s_full[gs & 1]);
            ++gs;
          }
          mma_commit(pv_done);
          if (n == cnt - 1) mma_commit(o_full);
          mma_commit(&kv_empty[sv]);
          if (more) mma_commit(&kv_empty[sk]);
          ++gp;
        }
      }
      // all MMAs issued by this thread must finish before TMEM is released
      mma_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0);
    }
  } else {
    // ================================================================ softmax + epilogue
    constexpr int KC = BS / 4;  // keys (S columns) per thread
    constexpr int OC = D / 4;   // O columns per thread
    const int cg = warp / 4, quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    const uint32_t t_oc = t_o0 + t_lane + cg * OC;
    float* xch = reinterpret_cast<float*>(smem + L::kXchOff);
    float* xsum = reinterpret_cast<float*>(smem + L::kSumOff);
    const float sl2 = g.scale * 1.4426950408889634f;
    int gstep = 0, ocons = 0;  // global step (= S buffer use / P / PV index)
    bool ok = true;
    // This thread's part of Q (row `row`, dims [cg*D/4, (cg+1)*D/4)) of the jj-th non-empty
    // item: from the 128-byte-swizzled staging tile into TMEM slot jj & 1 as bf16 pairs.
    auto copy_q = [&](int jj) -> bool {
      const int qb = jj % kQBufs, slot = jj & 1;
      bool w_ok = mbar_wait(&q_full[qb], (jj / kQBufs) & 1, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) return false;
      constexpr int DC = D / 4;
      const int d0 = cg * DC, half = d0 / 64, c0 = (d0 % 64) / 8;
      const unsigned char* tile = smem + L::kQOff + qb * L::kQBytes + half * (kTileM * 128) + row * 128;
      uint32_t w[DC / 2];
#pragma unroll
      for (int c = 0; c < DC / 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(tile + (((c0 + c) ^ (row & 7)) << 4));
        w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
      }
      const uint32_t dst = t_q0 + t_lane + slot * (D / 2) + cg * (DC / 2);
      if constexpr (DC == 32) tmem_st16(dst, w);
      else tmem_st8(dst, w);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&qt_full[slot]);
      mbar_arrive(&q_empty[qb]);
      return true;
    };
    int jq = -1;  // non-empty items started
    if (next_item(blockIdx.x) < p.n_items) ok = copy_q(0);
    int cnt_next = (int)blockIdx.x < p.n_items ? load_cnt(p, blockIdx.x) : 0;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const int cnt = cnt_next;  // the next item's count is fetched one item ahead
      cnt_next = item + (int)gridDim.x < p.n_items ? load_cnt(p, item + gridDim.x) : 0;
      const int i = item % g.NBq;
      // this row's query slot (rows >= BS belong to the tile's padding and are discarded)
      const bool qvalid = row < BS && row < query_block_nvalid(g, i);
      float* lse_row = p.lse + (size_t)item * BS;
      __nv_bfloat16* o_row = p.o + ((size_t)item * BS + row) * D + cg * OC;
      if (cnt == 0) {
        if (row < BS) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < OC / 8; ++c) reinterpret_cast<uint4*>(o_row)[c] = z;
          if (cg == 0) lse_row[row] = -INFINITY;
        }
        continue;
      }
      ++jq;
      const bool has_next = next_item(item + gridDim.x) < p.n_items;
      float m = -INFINITY, l = 0.f;
      // Key-block indices come 32 steps at a time (lane e holds step n0 + e), the next chunk's
      // load in flight while the current one runs; per chunk a ballot marks the steps whose
      // block is partial and each lane keeps its step's shape code, so no global load or
      // index arithmetic sits between a step's S and its P.
      int jnext = lane < cnt ? load_idx(p, item, lane) : 0;
      int nreg = BS;
      uint32_t partial = 0;
      for (int n = 0; n < cnt; ++n, ++gstep) {
        const int b = gstep & 1;
        if ((n & 31) == 0) {
          const int jcur = jnext;
          jnext = n + 32 + lane < cnt ? load_idx(p, item, n + 32 + lane) : 0;
          nreg = n + lane < cnt ? key_block_nvalid(g, jcur) : BS;
          partial = __ballot_sync(0xffffffffu, nreg < BS);
        }
        bool w_ok = mbar_wait(&s_full[b], (gstep >> 1) & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
        const uint32_t t_s = tmem_base + t_lane + b * 128;
        float s[KC];
        {
          uint32_t* sr = reinterpret_cast<uint32_t*>(s);
          if constexpr (KC == 32) tmem_ld32_wait(t_s + cg * KC, sr);
          else tmem_ld8_wait(t_s + cg * KC, sr);
        }
        // pad keys of a partial block get -inf (mask from the per-shape table)
        if ((partial >> (n & 31)) & 1u) {
          const int nv = __shfl_sync(0xffffffffu, nreg, n & 31) - cg * KC;
#pragma unroll
          for (int c = 0; c < KC; ++c)
            if (c >= nv) s[c] = -INFINITY;
        }
        float mx;
        {
          float a0 = s[0], a1 = s[1];
#pragma unroll
          for (int c = 2; c + 4 <= KC; c += 4) {
            a0 = max3f(a0, s[c], s[c + 1]);
            a1 = max3f(a1, s[c + 2], s[c + 3]);
          }
          mx = max3f(a0, a1, fmaxf(s[KC - 2], s[KC - 1]));
        }
        // exchange the four partial row maxima; the slots alternate with the step parity
        float* xs = xch + b * 512;
        xs[cg * 128 + row] = mx;
        named_bar_sync(1 + quarter, kSoftmaxThreads / 4);
        mx = fmaxf(fmaxf(xs[row], xs[128 + row]), fmaxf(xs[256 + row], xs[384 + row])) * sl2;
        // lazy rescale: raise the running max only when it grew by more than 8 (log2 units);
        // all four threads of a row take the same decision.  tcgen05.ld/st are warp-collective,
        // so a warp rescales together (alpha = 1 for rows that keep their max), after PV(n-1).
        const float m_new = (n == 0 || mx > m + 8.0f) ? mx : m;
        const bool resc = n > 0 && m_new != m;
        if (__any_sync(0xffffffffu, resc)) {
          bool pv_ok = mbar_wait(pv_done, (gstep - 1) & 1, abort_flag);
          pv_ok = __all_sync(0xffffffffu, pv_ok);
          if (!pv_ok) { ok = false; break; }
          tc_fence_after();
          const float alpha = resc ? fast_exp2(m - m_new) : 1.0f;
          l *= alpha;
          uint32_t r[OC];
          if constexpr (OC == 32) tmem_ld32_wait(t_oc, r);
          else tmem_ld16_wait(t_oc, r);
#pragma unroll
          for (int e = 0; e < OC; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          if constexpr (OC == 32) tmem_st32(t_oc, r);
          else tmem_st16(t_oc, r);
          tmem_wait_st();
        }
        m = m_new;
        // P = exp2(s * scale * log2e - m) as bf16 pairs into columns [cg*KC/2, ..) of this S
        // buffer (already read by every group: the exchange barrier above)
        const uint64_t sl2x2 = f2pack(sl2, sl2), nmx2 = f2pack(-m, -m);
        uint64_t sum2 = f2pack(0.f, 0.f);
        uint32_t pk[KC / 2];
#pragma unroll
        for (int e = 0; e < KC / 2; ++e) {
          float x0, x1;
          f2unpack(fma2(f2pack(s[2 * e], s[2 * e + 1]), sl2x2, nmx2), x0, x1);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          sum2 = add2(sum2, f2pack(p0, p1));
          pk[e] = pack_bf16x2(p0, p1);
        }
        if constexpr (KC == 32) tmem_st16(t_s + cg * (KC / 2), pk);
        else tmem_st4(t_s + cg * (KC / 2), pk);
        {
          float l0, l1;
          f2unpack(sum2, l0, l1);
          l += l0 + l1;
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
        // the next item's Q into the other slot (every S of the previous item, the slot's
        // last reader, completed before S(0) of this one)
        if (n == 0 && has_next && !copy_q(jq + 1)) { ok = false; break; }
      }
      if (!ok) break;
      // combine the four partial row sums
      xsum[cg * 128 + row] = l;
      named_bar_sync(1 + quarter, kSoftmaxThreads / 4);
      l = (xsum[row] + xsum[128 + row]) + (xsum[256 + row] + xsum[384 + row]);
      bool w_ok = mbar_wait(o_full, ocons & 1, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) { ok = false; break; }
      ++ocons;
      tc_fence_after();
      const float inv_l = qvalid ? 1.0f / l : 0.f;
      uint32_t r[OC];
      if constexpr (OC == 32) tmem_ld32_wait(t_oc, r);
      else tmem_ld16_wait(t_oc, r);
      if (row < BS) {
        uint4 v[OC / 8];
        uint32_t* v32 = reinterpret_cast<uint32_t*>(v);
#pragma unroll
        for (int e = 0; e < OC / 2; ++e)
          v32[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
#pragma unroll
        for (int e = 0; e < OC / 8; ++e) reinterpret_cast<uint4*>(o_row)[e] = v[e];
        if (cg == 0) lse_row[row] = qvalid ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, 512);
}

cudaError_t launch_fwd(const CUtensorMap* maps, const FwdParams& p, int n_sm, cudaStream_t s) {
  const int bs = p.g.BS, d = p.g.D;
  int grid = min(n_sm, p.n_items);
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
