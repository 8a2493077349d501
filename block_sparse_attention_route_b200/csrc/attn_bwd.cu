// attn_bwd.cu -- sparse flash-attention backward over the forward's selected blocks (sm_100a).
//
// Source: "LongCat-Video 高效長視頻生成探索世界模型的第壹步", section 2.2 (the sparse attention
// module ships forward and backward code for training and inference).  For the forward
// O = softmax(scale * Q K_S^T) V_S with LSE, and upstream gradient dO:
//   P = exp(scale * S - LSE),  dP = dO V^T,  Delta = rowsum(dO * O),  dS = P * (dP - Delta)
//   dV_j += P^T dO_i,  dK_j += scale * dS^T Q_i,  dQ_i += scale * dS K_j
// summed over every selected (query block i, key block j) pair.
//
// Four kernels, all on the caller's stream, no atomics (results are deterministic):
//   bwd_prep      Delta and log2-scaled LSE per query row (HBM-bound, one warp per row).
//   bwd_revidx    per (b, h): the key-block -> query-block index (CSR, lists ordered by i).
//   bwd_dkdv      key-major over current key blocks j: K_j, V_j stay in shared memory, the
//                 Q_i / dO_i tiles of the query blocks that selected j stream through a TMA
//                 ring; S^T and dP^T go to TMEM, P^T and dS^T (bf16) overwrite them and feed
//                 the dV / dK MMAs straight from TMEM; dV, dK accumulate in TMEM.
//   bwd_dq        query-major like the forward: Q_i, dO_i stay, K_j / V_j stream; S is double
//                 buffered so the next S and dP run on the tensor cores while the current
//                 dS is formed; dS (bf16) overwrites S and feeds dQ += dS K_j from TMEM.
// Splitting dQ from dK/dV costs two extra MMAs per pair (S and dP are recomputed) but needs
// no fp32 atomics, and the two 512-column TMEM plans fit exactly.
#include "common.cuh"

namespace bsa {

struct BwdWs {
  size_t ndelta, nlse2, rev_off, rev_list, order, ctr, total;
};
inline size_t bwd_align(size_t x) { return (x + 255) & ~size_t(255); }
BwdWs bwd_ws_layout(const Geo& g, int r) {
  BwdWs w;
  const size_t rows = (size_t)g.B * g.H * g.NBq * g.BS;
  w.ndelta = 0;
  w.nlse2 = bwd_align(rows * 4);
  w.rev_off = w.nlse2 + bwd_align(rows * 4);
  w.rev_list = w.rev_off + bwd_align((size_t)g.B * g.H * (g.NBk + 1) * 4);
  w.order = w.rev_list + bwd_align((size_t)g.B * g.H * g.NBq * r * 4);
  w.ctr = w.order + bwd_align((size_t)g.B * g.H * g.NBq * 4);
  w.total = w.ctr + 256;  // dK/dV work counter (one int, zeroed by the prep pass)
  return w;
}
struct BwdPtrs {
  const void *q, *k, *v, *kc, *vc, *o, *dO;
  const float* lse;
  const int *idx, *cnt;
  void *dq, *dk, *dv;
  char* ws;
};

struct BwdParams {
  Geo g;
  int r;
  int n_items;            // dkdv: B*H*NBq current key blocks; dq: B*H*NBq query blocks
  const int* idx;
  const int* cnt;
  const int* rev_off;     // [B*H][NBk+1]
  const int* rev_list;    // [B*H][NBq*r]
  const int* order;       // [B*H][NBq]: each head's current key blocks, longest list first
  const float* ndelta;    // [B*H*NBq*BS] -Delta
  const float* nlse2;     // [B*H*NBq*BS] -LSE * log2(e), -inf for pad rows
  int* ctr;               // dkdv: next item to hand out (minus gridDim.x), zeroed by prep
  __nv_bfloat16* out0;    // dkdv: dK, dq: dQ
  __nv_bfloat16* out1;    // dkdv: dV
};

// ------------------------------------------------------------------------------ prep
// ndelta = -rowsum(dO * O) and nlse2 = -LSE * log2(e) (-inf where LSE = -inf: pad rows or
// empty selections, so exp2(s + nlse2) = 0 there).  Stored negated so the elementwise passes
// form exp2(S * scale * log2e - LSE * log2e) and dP - Delta with single fused f32x2 ops.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dO,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ ndelta,
                                                       float* __restrict__ nlse2, size_t rows,
                                                       int* __restrict__ ctr) {
  constexpr int LPR = D / 8;  // lanes per row (16-byte vectors)
  if (blockIdx.x == 0 && threadIdx.x == 0) *ctr = 0;  // the dK/dV pass's work counter
  const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t row = t / LPR;
  const int c = (int)(t % LPR);
  float acc = 0.f;
  if (row < rows) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + c);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dO + row * D) + c);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(a2[e]), fb = __bfloat1622float2(b2[e]);
      acc = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc));
    }
  }
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && c == 0) {
    ndelta[row] = -acc;
    const float l = lse[row];
    nlse2[row] = (l == -INFINITY) ? -INFINITY : -l * 1.4426950408889634f;
  }
}

// ------------------------------------------------------------------------------ reverse index
// One CTA per (b, h) with kRevChunks warps; warp w owns a contiguous chunk of query blocks.
// (1) each warp counts, per key block, the selections in its chunk; (2) per key block the
// chunk counts are scanned, then the totals over key blocks, giving the CSR offsets and each
// chunk's first position in each list; (3) each warp fills its chunk's entries in increasing
// query-block order.  Lists come out ordered by i, deterministically and without atomics:
// the entries of one row are distinct blocks, so the lanes handling a row touch distinct
// counters.  (4) the head's current key blocks are ranked by decreasing list length into
// `order`, the key-major pass's hand-out order.
constexpr int kRevChunks = 8;
constexpr int kRevThreads = 32 * kRevChunks;
__global__ void __launch_bounds__(kRevThreads) bwd_revidx_kernel(const BwdParams p, int* rev_off,
                                                                int* rev_list, int* order) {
  // counts / cursors [kRevChunks][NBk], totals [NBk], scan scratch [kRevThreads]
  extern __shared__ int rsm[];
  const Geo& g = p.g;
  const int bh = blockIdx.x;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int* tot = rsm + kRevChunks * g.NBk;
  int* part = tot + g.NBk;
  for (int e = tid; e < kRevChunks * g.NBk; e += kRevThreads) rsm[e] = 0;
  __syncthreads();
  const int* idx = p.idx + (size_t)bh * g.NBq * p.r;
  const int* cnt = p.cnt + (size_t)bh * g.NBq;
  const int per_chunk = (g.NBq + kRevChunks - 1) / kRevChunks;
  const int i0 = warp * per_chunk, i1 = min(g.NBq, i0 + per_chunk);
  int* ck = rsm + warp * g.NBk;
  for (int i = i0; i < i1; ++i) {
    int c = cnt[i];
    if (c < 0 || c > p.r) { set_status(DEV_BAD_INDEX); c = min(max(c, 0), p.r); }
    for (int n = lane; n < c; n += 32) {
      const int j = idx[(size_t)i * p.r + n];
      if (j >= 0 && j < g.NBk) ck[j] += 1;
      else set_status(DEV_BAD_INDEX);
    }
    __syncwarp();
  }
  __syncthreads();
  const int per = (g.NBk + kRevThreads - 1) / kRevThreads;
  const int j0 = min(g.NBk, tid * per), j1 = min(g.NBk, j0 + per);
  int s_sum = 0;
  for (int j = j0; j < j1; ++j) {  // exclusive scan over the chunks of key block j
    int run = 0;
    for (int w = 0; w < kRevChunks; ++w) {
      const int v = rsm[w * g.NBk + j];
      rsm[w * g.NBk + j] = run;
      run += v;
    }
    tot[j] = run;
    s_sum += run;
  }
  part[tid] = s_sum;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int t = 0; t < kRevThreads; ++t) { const int v = part[t]; part[t] = run; run += v; }
  }
  __syncthreads();
  int run = part[tid];
  int* off = rev_off + (size_t)bh * (g.NBk + 1);
  for (int j = j0; j < j1; ++j) {  // list start of key block j; each chunk's first position
    off[j] = run;
    for (int w = 0; w < kRevChunks; ++w) rsm[w * g.NBk + j] += run;
    run += tot[j];
  }
  if (tid == kRevThreads - 1) off[g.NBk] = run;  // the last range ends at NBk: run = total
  __syncthreads();
  int* list = rev_list + (size_t)bh * g.NBq * p.r;
  const int cap = g.NBq * p.r;
  for (int i = i0; i < i1; ++i) {
    const int c = min(max(cnt[i], 0), p.r);
    for (int n = lane; n < c; n += 32) {
      const int j = idx[(size_t)i * p.r + n];
      if (j >= 0 && j < g.NBk) {
        const int pos = ck[j]++;
        if (pos < cap) list[pos] = i;
      }
    }
    __syncwarp();
  }
  // (4) the head's current key blocks by decreasing list length (a counting sort; blocks of
  // equal length in any order): the key-major pass hands its items out in this order within
  // each head, so the longest lists start first and the pass does not end on a long one
  __syncthreads();
  int* hist = rsm;  // [NBq + 1] over the chunk counters, which are no longer needed
  for (int e = tid; e <= g.NBq; e += kRevThreads) hist[e] = 0;
  __syncthreads();
  for (int jc = tid; jc < g.NBq; jc += kRevThreads) atomicAdd(&hist[min(tot[g.NBc + jc], g.NBq)], 1);
  __syncthreads();
  if (tid == 0) {
    int pos = 0;
    for (int len = g.NBq; len >= 0; --len) { const int v = hist[len]; hist[len] = pos; pos += v; }
  }
  __syncthreads();
  int* ord = order + (size_t)bh * g.NBq;
  for (int jc = tid; jc < g.NBq; jc += kRevThreads)
    ord[atomicAdd(&hist[min(tot[g.NBc + jc], g.NBq)], 1)] = jc;
}

// ------------------------------------------------------------------------------ common
// warps 0-15 elementwise: warp w reads TMEM lanes 32*(w%4).. and owns the 32-column group
// w/4 of every tile (S, dP: 4 x 32 columns); warp 16 TMA producer; warp 17 MMA issuer and
// TMEM owner.  No row reductions are needed in the backward (P comes from
// the stored LSE), so the column groups work independently: each writes its bf16 results
// back over TMEM columns it read itself, and the MMAs read the slices from where they land.
// Groups and quarters run independently:
// every arrive-counted mbarrier they signal is consumed before the MMA that lets any thread
// signal its next phase is issued, so no phase can be overrun.
constexpr int kBwdThreads = 576;
constexpr int kBwdProducer = 16, kBwdMma = 17, kBwdElem = 512;
constexpr int kBwdStages = 2;  // Q_i + dO_i stages of the key-major pass (64 KB each)
constexpr int kTile = 128;

// ------------------------------------------------------------------------------ dK / dV
// Work item = current key block (b, h, jc), jc in [0, NBq) (global id NBc + jc).  Steps =
// the query blocks that selected it, numbered globally (g) over the CTA's items.
// TMEM: R0 [0,128), R1 [128,256), dV [256,384), dK [384,512).  Step g computes S^T into
// R[g & 1] and dP^T into R[(g & 1) ^ 1]; the elementwise warps write P^T and dS^T (bf16) back
// over S^T in R[g & 1] -- each 32-column group over its own columns, as [P^T | dS^T] per 16
// queries (so the K16 slice kk of P^T sits at column 16kk, of dS^T at 16kk + 8) -- and
// R[(g & 1) ^ 1] is free once dP^T(g) has been loaded: S^T(g+1) goes there while P^T(g),
// dS^T(g) are being formed.
// MMA order: ... | dV(g-1) | S^T(g) | dK(g-1) | dP^T(g) | dV(g) | S^T(g+1) | ...; dP^T(g)
// reuses the region that dV(g-1) and dK(g-1) read, after them in issue order.
// Q_i and dO_i (with -lse2_i, -delta_i) share a 2-slot ring; a slot is released after dK(g),
// its last reader.
template <int BS, int D>
struct DkdvLayout {
  static constexpr int kKVBytes = BS * D * 2;      // K_j or V_j
  static constexpr int kTileBytes = BS * D * 2;    // Q_i or dO_i (BS query rows)
  static constexpr int kSlots = 2;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kKVBytes;
  static constexpr int kQOff = 2 * kKVBytes;                       // Q slots
  static constexpr int kDOOff = kQOff + kSlots * kTileBytes;      // dO slots
  static constexpr int kVecOff = kDOOff + kSlots * kTileBytes;    // -lse2 / -delta per Q slot
  static constexpr int kVecBytes = 2 * BS * 4;
  static constexpr int kBarOff = kVecOff + kSlots * kVecBytes;
  // kv_full, kv_empty, q_full[2], q_empty[2], s_full, dp_full, p_ready, dp_loaded, ds_ready,
  // acc_full, fin, iq_full[kQueue], iq_empty[kQueue]
  static constexpr int kQueue = 4;  // items handed from the producer to the other roles
  static constexpr int kNumBars = 2 + 2 * kSlots + 7 + 2 * kQueue;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kQueueOff = kMiscOff + 16;  // int [kQueue]
  static constexpr int kSlotNvOff = kQueueOff + kQueue * 4;  // int [kSlots]: valid queries
  static constexpr int kAlloc = kSlotNvOff + kSlots * 4 + 1024;
};

template <int BS, int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bsa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                        const BwdParams p) {
  using L = DkdvLayout<BS, D>;
  constexpr int NS = L::kSlots;
  static_assert(BS == 128, "the key-major pass maps one key row to one TMEM lane");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* kv_full = bars;           // K_j, V_j landed (one phase per non-empty item)
  uint64_t* kv_empty = bars + 1;      // K_j, V_j no longer needed
  uint64_t* q_full = bars + 2;        // [NS] Q_i, dO_i, -lse2_i, -delta_i landed in the slot
  uint64_t* q_empty = q_full + NS;    // [NS] slot free (after dK(g), the slot's last reader)
  uint64_t* s_full = q_empty + NS;    // S^T(g) in TMEM
  uint64_t* dp_full = s_full + 1;     // dP^T(g) in TMEM
  uint64_t* p_ready = dp_full + 1;    // P^T(g) (bf16) in TMEM (kBwdElem arrivals)
  uint64_t* dp_loaded = p_ready + 1;  // dP^T(g) read into registers (kBwdElem arrivals)
  uint64_t* ds_ready = dp_loaded + 1; // dS^T(g) (bf16) in TMEM (kBwdElem arrivals)
  uint64_t* acc_full = ds_ready + 1;  // dV and dK of the item complete
  uint64_t* fin_bar = acc_full + 1;
  uint64_t* iq_full = fin_bar + 1;            // [kQueue] queue entry written (producer)
  uint64_t* iq_empty = iq_full + L::kQueue;   // [kQueue] entry read by the MMA thread and
                                              // every elementwise thread
  volatile int* iq = reinterpret_cast<volatile int*>(smem + L::kQueueOff);
  // valid queries of the Q / dO tiles in each slot (written by the producer before the slot's
  // q_full arrival, read by the MMA thread after waiting on it)
  volatile int* slot_nv = reinterpret_cast<volatile int*>(smem + L::kSlotNvOff);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const Geo& g = p.g;

  if (tid == 0) {
    for (int k = 0; k < L::kQueue; ++k) {
      mbar_init(&iq_full[k], 1);
      mbar_init(&iq_empty[k], 1 + kBwdElem);
    }
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_ready, kBwdElem);
    mbar_init(dp_loaded, kBwdElem);
    mbar_init(ds_ready, kBwdElem);
    mbar_init(acc_full, 1);
    mbar_init(fin_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kBwdMma) { tmem_alloc(tmem_holder, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // item -> (bh, current key block jc); steps = rev list of global key block NBc + jc
  auto item_range = [&](int item, int& beg, int& end) {
    const int bh = item / g.NBq, jc = item % g.NBq;
    const int* off = p.rev_off + (size_t)bh * (g.NBk + 1) + g.NBc + jc;
    beg = off[0];
    end = off[1];
    if (beg < 0 || end < beg || end > g.NBq * p.r) { set_status(DEV_BAD_INDEX); beg = end = 0; }
  };
  // Work distribution: items (key blocks) are handed out dynamically, head by head and within
  // a head longest list first (the order the reverse index wrote) -- the first one per CTA
  // is queue position blockIdx.x, the rest come from a global counter -- so the CTAs finish
  // together although items differ in steps (a key block is selected by anything from a few
  // to a few hundred query blocks), and the CTAs running at once share one head's Q / dO.  The producer fetches,
  // zero-fills empty items itself, and passes the non-empty ones (then -1) to the MMA thread
  // and the elementwise warps through a small queue in shared memory.
  auto read_item = [&](int k, bool elem) -> int {  // k-th queue entry; -1 = no more
    const int slot = k % L::kQueue;
    bool w_ok = mbar_wait(&iq_full[slot], (k / L::kQueue) & 1, abort_flag);
    if (elem) w_ok = __all_sync(0xffffffffu, w_ok);
    if (!w_ok) return -1;
    const int it = iq[slot];
    mbar_arrive(&iq_empty[slot]);
    return it;
  };

  if (warp == kBwdProducer) {
    // ====================================================== TMA producer
    if (lane == 0) {
      int gq = 0, items = 0;        // steps, non-empty items
      int q_loads = 0;               // slot loads issued (for the drain)
      bool ok = true;
      for (int k = 0; ok; ++k) {
        // next non-empty item; empty ones get their zero dK / dV rows here.  Queue position
        // q is item (q / NBq) * NBq + order[q]: heads in turn, each head's longest lists first
        auto queue_item = [&](int q) -> int {
          if (q >= p.n_items) return p.n_items;
          int jc = p.order[q];
          if (jc < 0 || jc >= g.NBq) { set_status(DEV_BAD_INDEX); jc = 0; }
          return (q / g.NBq) * g.NBq + jc;
        };
        int item = queue_item(k == 0 ? (int)blockIdx.x : (int)gridDim.x + atomicAdd(p.ctr, 1));
        int beg = 0, end = 0;
        while (item < p.n_items) {
          item_range(item, beg, end);
          if (end > beg) break;
          const uint4 z = make_uint4(0, 0, 0, 0);
          uint4* dk4 = reinterpret_cast<uint4*>(p.out0 + (size_t)item * BS * D);
          uint4* dv4 = reinterpret_cast<uint4*>(p.out1 + (size_t)item * BS * D);
          for (int c = 0; c < BS * D / 8; ++c) { dk4[c] = z; dv4[c] = z; }
          item = queue_item((int)gridDim.x + atomicAdd(p.ctr, 1));
        }
        const int slot = k % L::kQueue;
        if (k >= L::kQueue && !mbar_wait(&iq_empty[slot], ((k / L::kQueue) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        iq[slot] = item < p.n_items ? item : -1;
        mbar_arrive(&iq_full[slot]);
        if (item >= p.n_items) break;
        const int bh = item / g.NBq, jc = item % g.NBq;
        // K_j, V_j for the item (once the previous item's S^T / dP^T MMAs released them)
        if (items > 0 && !mbar_wait(kv_empty, (items - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_expect_tx(kv_full, 2 * L::kKVBytes);
        const int krow = (bh * g.NBq + jc) * BS;
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          tma_load_2d(smem + L::kKOff + half * BS * 128, &tmK, half * 64, krow, kv_full);
          tma_load_2d(smem + L::kVOff + half * BS * 128, &tmV, half * 64, krow, kv_full);
        }
        ++items;
        const int* list = p.rev_list + (size_t)bh * g.NBq * p.r;
        for (int e = beg; e < end; ++e, ++gq) {
          int i = list[e];
          if (i < 0 || i >= g.NBq) { set_status(DEV_BAD_INDEX); i = 0; }
          const int slot = gq % NS, round = gq / NS;
          const int qrow = (bh * g.NBq + i) * BS;
          if (round > 0 && !mbar_wait(&q_empty[slot], (round - 1) & 1, abort_flag)) { ok = false; break; }
          unsigned char* vec = smem + L::kVecOff + slot * L::kVecBytes;
          slot_nv[slot] = query_block_nvalid(g, i);
          // whole tiles even for a partial query block (16-row boxes of only its valid rows
          // measured no faster)
          mbar_expect_tx(&q_full[slot], 2 * L::kTileBytes + L::kVecBytes);
#pragma unroll
          for (int half = 0; half < D / 64; ++half) {
            tma_load_2d(smem + L::kQOff + slot * L::kTileBytes + half * BS * 128, &tmQ, half * 64,
                        qrow, &q_full[slot]);
            tma_load_2d(smem + L::kDOOff + slot * L::kTileBytes + half * BS * 128, &tmdO, half * 64,
                        qrow, &q_full[slot]);
          }
          bulk_load(vec, p.nlse2 + (size_t)qrow, BS * 4, &q_full[slot]);
          bulk_load(vec + BS * 4, p.ndelta + (size_t)qrow, BS * 4, &q_full[slot]);
          ++q_loads;
        }
      }
      // drain every copy still in flight
      for (int s = 0; s < NS; ++s) {
        const int ql = q_loads / NS + (s < q_loads % NS ? 1 : 0);
        if (ql > 0) mbar_wait_drain(&q_full[s], (ql - 1) & 1);
      }
      if (items > 0) mbar_wait_drain(kv_full, (items - 1) & 1);
    }
  } else if (warp == kBwdMma) {
    // ====================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idTS = idesc_bf16(kTile, D, 0, 1);    // dV, dK: B MN-major
      // queries of step g on the tensor cores: the query block's valid prefix rounded up to
      // 16 (the MMA's N step), so a partial block's S^T, dP^T (N) and dV, dK (K) shrink with
      // it; read from the slot when S^T(g) is issued and kept for the step's other MMAs
      int nq_even = BS, nq_odd = BS;  // for steps g with g & 1 == 0 / 1
      auto nq_step = [&](int gg) -> int { return (gg & 1) ? nq_odd : nq_even; };
      const uint64_t dK0 = smem_desc_sw128(smem_u32(smem + L::kKOff), 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(smem_u32(smem + L::kVOff), 16, 1024);
      const uint64_t dQk = smem_desc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
      const uint64_t dOk = smem_desc_sw128(smem_u32(smem + L::kDOOff), 16, 1024);
      const uint64_t dQmn = smem_desc_sw128(smem_u32(smem + L::kQOff), BS * 128, 1024);
      const uint64_t dOmn = smem_desc_sw128(smem_u32(smem + L::kDOOff), BS * 128, 1024);
      const uint32_t t_dv = tmem_base + 256, t_dk = tmem_base + 384;
      static_assert(NS == 2, "slot = step & 1");
      int kv_items = 0;  // K/V loads waited for
      bool ok = true;
      // S^T(g) = K Q^T into R[g & 1]; the first step of an item waits for the item's K/V
      auto issue_S = [&](int gg, bool item_first) -> bool {
        if (item_first) {
          if (!mbar_wait(kv_full, kv_items & 1, abort_flag)) return false;
          ++kv_items;
        }
        if (!mbar_wait(&q_full[gg & 1], (gg >> 1) & 1, abort_flag)) return false;
        tc_fence_after();
        {
          const int nv = slot_nv[gg & 1];
          const int nq = nv >= BS ? BS : (nv <= 16 ? 16 : (nv + 15) & ~15);
          if (gg & 1) nq_odd = nq;
          else nq_even = nq;
        }
        const uint32_t idSS = idesc_bf16(kTile, nq_step(gg), 0, 0);  // both K-major
        const uint64_t rq = dQk + (uint64_t)(((gg & 1) * L::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4;
          mma_ss(tmem_base + (gg & 1) * 128, dK0 + off, rq + off, idSS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
        return true;
      };
      // dP^T(g) = V dO^T into R[(g & 1) ^ 1] (dO landed with Q: issue_S(g) waited for the
      // slot); after an item's last one K_j, V_j are free
      auto issue_dP = [&](int gg, bool item_last) -> bool {
        const uint64_t rdo = dOk + (uint64_t)(((gg & 1) * L::kTileBytes) >> 4);
        const uint32_t idSS = idesc_bf16(kTile, nq_step(gg), 0, 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4;
          mma_ss(tmem_base + ((gg & 1) ^ 1) * 128, dV0 + off, rdo + off, idSS, kk > 0 ? 1u : 0u);
        }
        mma_commit(dp_full);
        if (item_last) mma_commit(kv_empty);
        return true;
      };
      // dV(g) += P^T(g) dO or dK(g) += dS^T(g) Q; the K16 slice kk of P^T sits at column
      // 32*(kk/2) + 8*(kk%2) of R[g & 1], of dS^T 16 columns further
      auto issue_grad = [&](int gg, bool item_first, bool is_dk) {
        const uint32_t r = tmem_base + (gg & 1) * 128 + (is_dk ? 16 : 0);
        const uint64_t mb = (is_dk ? dQmn : dOmn) + (uint64_t)(((gg & 1) * L::kTileBytes) >> 4);
        const uint32_t acc_d = is_dk ? t_dk : t_dv;
        const int nk = nq_step(gg) / 16;
#pragma unroll
        for (int kk = 0; kk < BS / 16; ++kk)
          if (kk < nk)
            mma_ts(acc_d, r + 32 * (kk >> 1) + 8 * (kk & 1), mb + (uint64_t)((kk * 2048) >> 4),
                   idTS, (item_first && kk == 0) ? 0u : 1u);
      };
      // Per step g: dV(g) | S^T(g+1) (into the region dP^T(g) left) | dK(g) | dP^T(g+1) (into
      // the region dV(g), dK(g) just read).  The elementwise warps form P^T(g+1) while the
      // tensor cores run dK(g) and dP^T(g+1).  The first step of an item is issued at the end
      // of the previous item's last step (its S^T waits for the item's K/V).
      int beg = 0, end = 0, kq = 0;
      int item = read_item(kq++, false);
      int gg = 0;
      if (item >= 0) {
        item_range(item, beg, end);
        ok = issue_S(0, true) && issue_dP(0, end - beg == 1);
      }
      while (item >= 0 && ok) {
        int nitem = -1, nbeg = 0, nend = 0;
        for (int e = beg; e < end; ++e, ++gg) {
          const bool first = e == beg, more = e + 1 < end;
          if (!mbar_wait(p_ready, gg & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_grad(gg, first, false);
          if (more) {
            if (!mbar_wait(dp_loaded, gg & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (!issue_S(gg + 1, false)) { ok = false; break; }
          }
          if (!mbar_wait(ds_ready, gg & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_grad(gg, first, true);
          mma_commit(&q_empty[gg & 1]);
          if (more) {
            if (!issue_dP(gg + 1, e + 2 == end)) { ok = false; break; }
          } else {
            mma_commit(acc_full);
            nitem = read_item(kq++, false);  // the next item, looked up at this item's end
            if (nitem >= 0) {
              item_range(nitem, nbeg, nend);
              if (!mbar_wait(dp_loaded, gg & 1, abort_flag)) { ok = false; break; }
              tc_fence_after();
              if (!issue_S(gg + 1, true) || !issue_dP(gg + 1, nend - nbeg == 1)) { ok = false; break; }
            }
          }
        }
        item = nitem;
        beg = nbeg;
        end = nend;
      }
      mma_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0);
    }
  } else if (warp < kBwdElem / 32) {
    // ====================================================== elementwise + epilogue
    const int row = 32 * (warp % 4) + lane;  // key slot within the block
    const int cg = warp / 4;                 // 32-column group
    const uint32_t t_lane = (uint32_t)(32 * (warp % 4)) << 16;
    const uint32_t t_dv = tmem_base + t_lane + 256, t_dk = tmem_base + t_lane + 384;
    const float sl2 = g.scale * 1.4426950408889634f;
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    int gs = 0, items = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = read_item(k, true);
      if (item < 0) break;
      int beg, end;
      item_range(item, beg, end);
      const int jc = item % g.NBq;
      const bool kvalid = row < query_block_nvalid(g, jc);  // key slot in the valid prefix
      for (int e = beg; e < end; ++e, ++gs) {
        // valid queries of this step's query block, from its slot (the slot's q_full phase
        // for this step has completed: S^T(g) was issued after it), so a group whose 32 query
        // columns all lie past a partial block's valid prefix can skip the step: the tensor
        // cores compute and read only the first roundup16(valid) columns
        {
          bool w_ok = mbar_wait(&q_full[gs % NS], (gs / NS) & 1, abort_flag);
          w_ok = __all_sync(0xffffffffu, w_ok);
          if (!w_ok) { ok = false; break; }
        }
        if (cg * 32 >= slot_nv[gs % NS]) {
          // nothing to form: keep the waits and arrivals in order
          bool w_ok = mbar_wait(s_full, gs & 1, abort_flag);
          w_ok = __all_sync(0xffffffffu, w_ok);
          if (!w_ok) { ok = false; break; }
          mbar_arrive(p_ready);
          w_ok = mbar_wait(dp_full, gs & 1, abort_flag);
          w_ok = __all_sync(0xffffffffu, w_ok);
          if (!w_ok) { ok = false; break; }
          mbar_arrive(dp_loaded);
          mbar_arrive(ds_ready);
          continue;
        }
        // this group's 32 query columns of step g: P^T = exp2(S^T*sl2 - lse2[q]) as soon as
        // S^T is in, then dS^T = P^T * (dP^T - delta[q]) once dP^T is; both in bf16 back over
        // the group's own S^T columns as [P^T 16 cols | dS^T 16 cols]
        const uint32_t rx = tmem_base + t_lane + (gs & 1) * 128;
        const uint32_t ry = tmem_base + t_lane + ((gs & 1) ^ 1) * 128;
        const float* vec = reinterpret_cast<const float*>(smem + L::kVecOff + (gs % NS) * L::kVecBytes);
        const float4* nl4 = reinterpret_cast<const float4*>(vec + cg * 32);       // -lse2[q]
        const float4* nd4 = reinterpret_cast<const float4*>(vec + BS + cg * 32);  // -delta[q]
        bool w_ok = mbar_wait(s_full, gs & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
        float pf[32];
        {
          uint32_t* sr = reinterpret_cast<uint32_t*>(pf);
          tmem_ld32_wait(rx + cg * 32, sr);
          if (!kvalid) {  // pad key slot: S^T = -inf, so P^T = dS^T = 0
#pragma unroll
            for (int c = 0; c < 32; ++c) pf[c] = -INFINITY;
          }
          uint32_t pk[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const float4 nl = nl4[e4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int e2 = 2 * e4 + h;
              float x0, x1;
              f2unpack(fma2(f2pack(pf[2 * e2], pf[2 * e2 + 1]), sl2x2,
                            h ? f2pack(nl.z, nl.w) : f2pack(nl.x, nl.y)), x0, x1);
              pf[2 * e2] = fast_exp2(x0);
              pf[2 * e2 + 1] = fast_exp2(x1);
              pk[e2] = pack_bf16x2(pf[2 * e2], pf[2 * e2 + 1]);
            }
          }
          tmem_st16(rx + cg * 32, pk);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(p_ready);  // dV(g) may start
        }
        w_ok = mbar_wait(dp_full, gs & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int round = 0; round < 2; ++round) {
          uint32_t dr[16], dk[8];
          tmem_ld16_wait(ry + cg * 32 + round * 16, dr);
          if (round == 1) {
            tc_fence_before();
            mbar_arrive(dp_loaded);  // R[(g & 1) ^ 1] may now take S^T(g+1)
          }
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4) {
            const float4 nd = nd4[round * 4 + e4];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int j = 2 * e4 + h;         // column pair within the round
              const int e2 = round * 8 + j;     // column pair within the 32
              float s0, s1;
              f2unpack(mul2(f2pack(pf[2 * e2], pf[2 * e2 + 1]),
                            add2(f2pack(__uint_as_float(dr[2 * j]), __uint_as_float(dr[2 * j + 1])),
                                 h ? f2pack(nd.z, nd.w) : f2pack(nd.x, nd.y))),
                       s0, s1);
              dk[j] = pack_bf16x2(s0, s1);
            }
          }
          tmem_st8(rx + cg * 32 + 16 + round * 8, dk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ds_ready);  // dK(g) may start
      }
      if (!ok) break;
      // epilogue: dV, dK rows of this key block (zeros for pad keys)
      const size_t orow = (size_t)item * BS + row;
      __nv_bfloat16* dv_row = p.out1 + orow * D;
      __nv_bfloat16* dk_row = p.out0 + orow * D;
      bool w_ok = mbar_wait(acc_full, items & 1, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) { ok = false; break; }
      ++items;
      tc_fence_after();
      constexpr int DC = D / 4;  // dV / dK columns of this group, 16 at a time
#pragma unroll
      for (int c0 = 0; c0 < DC; c0 += 16) {
#pragma unroll
        for (int which = 0; which < 2; ++which) {  // dV, then dK (scaled)
          uint32_t a[16];
          tmem_ld16_wait((which ? t_dk : t_dv) + cg * DC + c0, a);
          const float sc = which ? g.scale : 1.0f;
          uint4 va[2];
          uint32_t* a32 = reinterpret_cast<uint32_t*>(va);
#pragma unroll
          for (int e2 = 0; e2 < 8; ++e2)
            a32[e2] = kvalid ? pack_bf16x2(__uint_as_float(a[2 * e2]) * sc, __uint_as_float(a[2 * e2 + 1]) * sc)
                             : 0u;
          __nv_bfloat16* dst = (which ? dk_row : dv_row) + cg * DC + c0;
          reinterpret_cast<uint4*>(dst)[0] = va[0];
          reinterpret_cast<uint4*>(dst)[1] = va[1];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwdMma) tmem_dealloc(tmem_base, 512);
}

// ------------------------------------------------------------------------------ dQ
// Work item = query block (b, h, i); steps = its selected key blocks (cached ones included).
// TMEM: Q [0,64) and dO [64,128) as bf16 pairs (A operands, copied in by the elementwise warps
// from the TMA-staged tiles once per item), S [128,256), dP [256,384), dQ [384,512).  dS (bf16)
// goes back over dP, each 32-key group's 16 columns over the first half of its own dP columns,
// and feeds dQ += dS K_n from TMEM.  All three MMAs read one operand from TMEM, so per pair
// shared memory serves only the K / V tiles.  MMA order per step n: S(n+1) (once S(n) was read
// out) | dQ(n), dP(n+1) (once dS(n) is in): the exponentials of step n+1 run while the tensor
// cores do dQ(n) and dP(n+1).
template <int BS, int D>
struct DqLayout {
  static constexpr int kTileBytes = kTile * D * 2;  // Q_i / dO_i staging (128-row tiles)
  static constexpr int kKVBytes = BS * D * 2;
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kTileBytes;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kStages = 5;
  static constexpr int kBarOff = kRingOff + kStages * kKVBytes;
  // q_full, q_empty, kv_full[5], kv_empty[5], s_full, s_loaded, dp_full, ds_full, dq_full, fin
  static constexpr int kNumBars = 2 + 2 * kStages + 6;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kAlloc = kMiscOff + 16 + 1024;
};

template <int BS, int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bsa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmVc,
                      const BwdParams p) {
  using L = DqLayout<BS, D>;
  constexpr int S = L::kStages;
  static_assert(BS == 128, "dS of one row fills the 32-key groups of a 128-key block");
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* q_full = bars;            // Q_i, dO_i staged in shared memory
  uint64_t* q_empty = bars + 1;       // ... and copied into TMEM (kBwdElem arrivals); the MMA
                                      // thread waits on it too before the item's first S
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = kv_full + S;
  uint64_t* s_full = kv_empty + S;    // S(n) in TMEM
  uint64_t* s_loaded = s_full + 1;    // S(n) read out (kBwdElem arrivals)
  uint64_t* dp_full = s_loaded + 1;   // dP(n) in TMEM
  uint64_t* ds_full = dp_full + 1;    // dS(n) in TMEM (kBwdElem arrivals)
  uint64_t* dq_full = ds_full + 1;    // dQ of the item complete
  uint64_t* fin_bar = dq_full + 1;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscOff + 4);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const Geo& g = p.g;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, kBwdElem);
    for (int s = 0; s < S; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    mbar_init(s_full, 1);
    mbar_init(s_loaded, kBwdElem);
    mbar_init(dp_full, 1);
    mbar_init(ds_full, kBwdElem);
    mbar_init(dq_full, 1);
    mbar_init(fin_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kBwdMma) { tmem_alloc(tmem_holder, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  constexpr uint32_t kTq = 0, kTdo = 64, kTs = 128, kTdp = 256, kTdq = 384;  // TMEM columns

  auto item_cnt = [&](int item) {
    int c = __ldg(p.cnt + item);
    if (c < 0 || c > p.r) { set_status(DEV_BAD_INDEX); c = min(max(c, 0), p.r); }
    return c;
  };
  auto item_idx = [&](int item, int n) {
    int j = __ldg(p.idx + (size_t)item * p.r + n);
    if (j < 0 || j >= g.NBk) { set_status(DEV_BAD_INDEX); j = 0; }
    return j;
  };

  if (warp == kBwdProducer) {
    // ====================================================== TMA producer: per step K_n, V_n
    if (lane == 0) {
      int seq = 0, qloads = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const int cnt = item_cnt(item);
        if (cnt == 0) continue;
        if (qloads > 0 && !mbar_wait(q_empty, (qloads - 1) & 1, abort_flag)) { ok = false; break; }
        mbar_expect_tx(q_full, 2 * L::kTileBytes);
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          tma_load_2d(smem + L::kQOff + half * kTile * 128, &tmQ, half * 64, item * BS, q_full);
          tma_load_2d(smem + L::kDOOff + half * kTile * 128, &tmdO, half * 64, item * BS, q_full);
        }
        ++qloads;
        const int bhx = item / g.NBq;
        for (int n = 0; n < cnt && ok; ++n) {
          const int j = item_idx(item, n);
          const CUtensorMap *mk, *mv;
          int row;
          if (j < g.NBc) { mk = &tmKc; mv = &tmVc; row = (bhx * g.NBc + j) * BS; }
          else { mk = &tmK; mv = &tmV; row = (bhx * g.NBq + (j - g.NBc)) * BS; }
          for (int t = 0; t < 2; ++t) {  // K_n then V_n
            const int stage = seq % S, round = seq / S;
            if (round > 0 && !mbar_wait(&kv_empty[stage], (round - 1) & 1, abort_flag)) { ok = false; break; }
            unsigned char* dst = smem + L::kRingOff + stage * L::kKVBytes;
            mbar_expect_tx(&kv_full[stage], L::kKVBytes);
#pragma unroll
            for (int half = 0; half < D / 64; ++half)
              tma_load_2d(dst + half * BS * 128, t == 0 ? mk : mv, half * 64, row, &kv_full[stage]);
            ++seq;
          }
        }
      }
      for (int st = 0; st < S; ++st) {
        const int loads = seq / S + (st < seq % S ? 1 : 0);
        if (loads > 0) mbar_wait_drain(&kv_full[st], (loads - 1) & 1);
      }
      if (qloads > 0) mbar_wait_drain(q_full, (qloads - 1) & 1);
    }
  } else if (warp == kBwdMma) {
    // ====================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kTile, BS, 0, 0);   // S, dP: B (K or V tile) K-major
      constexpr uint32_t idQ = idesc_bf16(kTile, D, 0, 1);    // dQ: B (K tile) MN-major
      const uint64_t dk = smem_desc_sw128(smem_u32(smem + L::kRingOff), 16, 1024);
      const uint64_t dkmn = smem_desc_sw128(smem_u32(smem + L::kRingOff), BS * 128, 1024);
      int items = 0, gn = 0;  // non-empty items, global step
      bool ok = true;
      // the ring holds K_n at seq_base + 2n and V_n at seq_base + 2n + 1
      int seq_base = 0;
      auto wait_tile = [&](int seq) -> bool {
        if (!mbar_wait(&kv_full[seq % S], (seq / S) & 1, abort_flag)) return false;
        tc_fence_after();
        return true;
      };
      auto mma_S = [&](int n) {  // S(n) = Q K_n^T (A = Q from TMEM)
        const uint64_t kb = dk + (uint64_t)((((seq_base + 2 * n) % S) * L::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = ((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4;
          mma_ts(tmem_base + kTs, tmem_base + kTq + kk * 8, kb + offk, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_full);
      };
      auto mma_dP = [&](int n) {  // dP(n) = dO V_n^T (A = dO from TMEM); then V_n is done
        const int seq = seq_base + 2 * n + 1;
        const uint64_t vb = dk + (uint64_t)(((seq % S) * L::kKVBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = ((kk / 4) * (BS * 128) + (kk % 4) * 32) >> 4;
          mma_ts(tmem_base + kTdp, tmem_base + kTdo + kk * 8, vb + offk, idS, kk > 0 ? 1u : 0u);
        }
        mma_commit(&kv_empty[seq % S]);
        mma_commit(dp_full);
      };
      for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        const int cnt = item_cnt(item);
        if (cnt == 0) continue;
        // Q, dO of the item in TMEM (the previous item's S / dP MMAs were issued before, and
        // the elementwise warps copy them only after reading that item's last S / dP)
        if (!mbar_wait(q_empty, items & 1, abort_flag)) { ok = false; break; }
        ++items;
        // S(0) into S once the previous step's S was read out; dP(0) into dP after the previous
        // dQ (issue order)
        if (gn > 0 && !mbar_wait(s_loaded, (gn - 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        if (!wait_tile(seq_base) || !wait_tile(seq_base + 1)) { ok = false; break; }
        mma_S(0);
        mma_dP(0);
        for (int n = 0; n < cnt && ok; ++n, ++gn) {
          const bool more = n + 1 < cnt;
          if (more) {  // S(n+1) once S(n) was read out
            if (!mbar_wait(s_loaded, gn & 1, abort_flag)) { ok = false; break; }
            tc_fence_after();
            if (!wait_tile(seq_base + 2 * (n + 1))) { ok = false; break; }
            mma_S(n + 1);
            if (!wait_tile(seq_base + 2 * (n + 1) + 1)) { ok = false; break; }  // V_{n+1}, early
          }
          // dQ += dS(n) K_n (A = dS over the dP columns), then dP(n+1) into those columns
          if (!mbar_wait(ds_full, gn & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const int kseq = seq_base + 2 * n;
          const uint64_t kb = dkmn + (uint64_t)(((kseq % S) * L::kKVBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BS / 16; ++kk)  // dS of keys [16kk, 16kk+16): group kk/2's columns
            mma_ts(tmem_base + kTdq, tmem_base + kTdp + 32 * (kk >> 1) + 8 * (kk & 1),
                   kb + (uint64_t)((kk * 2048) >> 4), idQ, (n > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&kv_empty[kseq % S]);  // K_n done
          if (more) mma_dP(n + 1);
        }
        if (!ok) break;
        mma_commit(dq_full);
        seq_base += 2 * cnt;
      }
      mma_commit(fin_bar);
      mbar_wait_drain(fin_bar, 0);
    }
  } else if (warp < kBwdElem / 32) {
    // ====================================================== elementwise + epilogue
    const int quarter = warp % 4;
    const int row = 32 * quarter + lane;     // query row of the 128-row tile
    const int cg = warp / 4;                 // 32-column group (BS / 4 keys, D / 4 dims)
    const uint32_t t_lane = (uint32_t)(32 * quarter) << 16;
    const uint32_t t_s = tmem_base + t_lane + kTs, t_dp = tmem_base + t_lane + kTdp;
    const uint32_t t_dq = tmem_base + t_lane + kTdq;
    const float sl2 = g.scale * 1.4426950408889634f;
    constexpr int KC = BS / 4;
    int qc = 0, gn = 0, dqc = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      const int cnt = item_cnt(item);
      const size_t qrow = (size_t)item * BS + row;
      __nv_bfloat16* dq_row = p.out0 + qrow * D;
      if (cnt == 0) {
        if (row < BS) {
          const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int c = 0; c < D / 32; ++c) reinterpret_cast<uint4*>(dq_row + cg * (D / 4))[c] = z;
        }
        continue;
      }
      // Q and dO rows of this thread (dims [D/4*cg, D/4*(cg+1))) from the 128-byte-swizzled
      // staging tiles into TMEM as bf16 pairs: the A operands of S and dP
      {
        bool w_ok = mbar_wait(q_full, qc & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        ++qc;
        constexpr int DC = D / 4;         // dims of this group: DC / 8 chunks of 16 bytes
        const int d0 = cg * DC, half = d0 / 64, c0 = (d0 % 64) / 8;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const unsigned char* tile = smem + (t ? L::kDOOff : L::kQOff) + half * (kTile * 128) + row * 128;
          uint32_t w[DC / 2];
#pragma unroll
          for (int c = 0; c < DC / 8; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + (((c0 + c) ^ (row & 7)) << 4));
            w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
          }
          const uint32_t dst = tmem_base + t_lane + (t ? kTdo : kTq) + cg * (DC / 2);
          if constexpr (DC == 32) tmem_st16(dst, w);
          else tmem_st8(dst, w);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(q_empty);  // staging free; Q, dO in TMEM
      }
      const float nl2 = row < BS ? p.nlse2[qrow] : -INFINITY;  // -inf: pad row -> P = 0
      const float nd = row < BS ? p.ndelta[qrow] : 0.f;
      const uint64_t nl2x2 = f2pack(nl2, nl2), ndx2 = f2pack(nd, nd), sl2x2 = f2pack(sl2, sl2);
      // key-block indices 32 steps at a time, the next chunk's load in flight; per chunk a
      // ballot of the partial blocks and each lane's shape code (as in the forward)
      int jnext = lane < cnt ? item_idx(item, lane) : 0;
      int nreg = BS;
      uint32_t partial = 0;
      for (int n = 0; n < cnt; ++n, ++gn) {
        if ((n & 31) == 0) {
          const int jcur = jnext;
          jnext = n + 32 + lane < cnt ? item_idx(item, n + 32 + lane) : 0;
          nreg = n + lane < cnt ? key_block_nvalid(g, jcur) : BS;
          partial = __ballot_sync(0xffffffffu, nreg < BS);
        }
        // P = exp2(S*sl2 - lse2) for this group's KC keys as soon as S(n) is in
        bool w_ok = mbar_wait(s_full, gn & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
        float pf[KC];
        tmem_ld32_wait(t_s + cg * KC, reinterpret_cast<uint32_t*>(pf));
        tc_fence_before();
        mbar_arrive(s_loaded);  // S may take S(n+1)
        if ((partial >> (n & 31)) & 1u) {  // pad keys (slots >= the valid count): P = 0
          const int nv = __shfl_sync(0xffffffffu, nreg, n & 31) - cg * KC;
#pragma unroll
          for (int c = 0; c < KC; ++c)
            if (c >= nv) pf[c] = -INFINITY;
        }
#pragma unroll
        for (int e2 = 0; e2 < KC / 2; ++e2) {
          float x0, x1;
          f2unpack(fma2(f2pack(pf[2 * e2], pf[2 * e2 + 1]), sl2x2, nl2x2), x0, x1);
          pf[2 * e2] = fast_exp2(x0);
          pf[2 * e2 + 1] = fast_exp2(x1);
        }
        // dS = P (dP - delta) once dP(n) is in, back over this group's own dP columns as
        // bf16 pairs (keys [KC*cg, KC*cg + KC) at columns [KC*cg, KC*cg + KC/2)), 16 at a time
        w_ok = mbar_wait(dp_full, gn & 1, abort_flag);
        w_ok = __all_sync(0xffffffffu, w_ok);
        if (!w_ok) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int round = 0; round < 2; ++round) {
          uint32_t dr[16], pk[8];
          tmem_ld16_wait(t_dp + cg * KC + round * 16, dr);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int e2 = round * 8 + j;
            float s0, s1;
            f2unpack(mul2(f2pack(pf[2 * e2], pf[2 * e2 + 1]),
                          add2(f2pack(__uint_as_float(dr[2 * j]), __uint_as_float(dr[2 * j + 1])), ndx2)),
                     s0, s1);
            pk[j] = pack_bf16x2(s0, s1);
          }
          tmem_st8(t_dp + cg * KC + round * 8, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ds_full);  // dQ(n) may start
      }
      if (!ok) break;
      bool w_ok = mbar_wait(dq_full, dqc & 1, abort_flag);
      w_ok = __all_sync(0xffffffffu, w_ok);
      if (!w_ok) { ok = false; break; }
      ++dqc;
      tc_fence_after();
      {
        constexpr int DC = D / 4;
        uint32_t a[DC];
        if constexpr (DC == 32) tmem_ld32_wait(t_dq + cg * DC, a);
        else tmem_ld16_wait(t_dq + cg * DC, a);
        if (row < BS) {
          uint4 v[DC / 8];
          uint32_t* v32 = reinterpret_cast<uint32_t*>(v);
#pragma unroll
          for (int e2 = 0; e2 < DC / 2; ++e2)
            v32[e2] = (nl2 == -INFINITY) ? 0u
                                         : pack_bf16x2(__uint_as_float(a[2 * e2]) * g.scale,
                                                       __uint_as_float(a[2 * e2 + 1]) * g.scale);
#pragma unroll
          for (int e2 = 0; e2 < DC / 8; ++e2) reinterpret_cast<uint4*>(dq_row + cg * DC)[e2] = v[e2];
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kBwdMma) tmem_dealloc(tmem_base, 512);
}

// ------------------------------------------------------------------------------ host side
// maps: 0 Q (box 128 rows), 1 K, 2 V, 3 K cache, 4 V cache (box BS rows), 5 dO (box 128 rows)
bsa_status_t run_bwd(const Geo& g, int r, const BwdPtrs& P, const BwdWs& w, const CUtensorMap* maps,
                     int n_sm, cudaStream_t s) {
  if (g.BS != 128) return BSA_ERR_UNSUPPORTED;  // the key-major pass needs 128-token blocks
  float* ndelta = reinterpret_cast<float*>(P.ws + w.ndelta);
  float* nlse2 = reinterpret_cast<float*>(P.ws + w.nlse2);
  int* rev_off = reinterpret_cast<int*>(P.ws + w.rev_off);
  int* rev_list = reinterpret_cast<int*>(P.ws + w.rev_list);
  int* order = reinterpret_cast<int*>(P.ws + w.order);
  int* ctr = reinterpret_cast<int*>(P.ws + w.ctr);
  const size_t rows = (size_t)g.B * g.H * g.NBq * g.BS;
  {
    const size_t threads = rows * (g.D / 8);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    if (g.D == 128)
      bwd_prep_kernel<128><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(P.o),
                                                  static_cast<const __nv_bfloat16*>(P.dO), P.lse,
                                                  ndelta, nlse2, rows, ctr);
    else
      bwd_prep_kernel<64><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(P.o),
                                                 static_cast<const __nv_bfloat16*>(P.dO), P.lse,
                                                 ndelta, nlse2, rows, ctr);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  BwdParams bp;
  bp.g = g;
  bp.r = r;
  bp.n_items = g.B * g.H * g.NBq;
  bp.idx = P.idx;
  bp.cnt = P.cnt;
  bp.rev_off = rev_off;
  bp.rev_list = rev_list;
  bp.order = order;
  bp.ndelta = ndelta;
  bp.nlse2 = nlse2;
  bp.ctr = ctr;
  {
    const size_t smem = (size_t)((kRevChunks + 1) * g.NBk + kRevThreads) * 4;
    if (cudaFuncSetAttribute(bwd_revidx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return BSA_ERR_CUDA;
    bwd_revidx_kernel<<<g.B * g.H, kRevThreads, smem, s>>>(bp, rev_off, rev_list, order);
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;
  }
  const int grid = max(1, min(n_sm, bp.n_items));
#define BSA_LAUNCH_BWD(Dv)                                                                        \
  do {                                                                                            \
    BwdParams a = bp;                                                                             \
    a.out0 = static_cast<__nv_bfloat16*>(P.dk);                                                   \
    a.out1 = static_cast<__nv_bfloat16*>(P.dv);                                                   \
    auto k1 = bsa_bwd_dkdv_kernel<128, Dv>;                                                       \
    const int s1 = DkdvLayout<128, Dv>::kAlloc;                                                   \
    if (cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, s1) != cudaSuccess) \
      return BSA_ERR_CUDA;                                                                        \
    cudaEvent_t e1;                                                                               \
    const int w1 = timed_begin(BSA_TIMED_BWD_DKDV, s, &e1);                                       \
    k1<<<grid, kBwdThreads, s1, s>>>(maps[1], maps[2], maps[0], maps[5], a);                      \
    timed_end(w1, s, e1);                                                                         \
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;                                   \
    BwdParams c = bp;                                                                             \
    c.out0 = static_cast<__nv_bfloat16*>(P.dq);                                                   \
    c.out1 = nullptr;                                                                             \
    auto k2 = bsa_bwd_dq_kernel<128, Dv>;                                                         \
    const int s2 = DqLayout<128, Dv>::kAlloc;                                                     \
    if (cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, s2) != cudaSuccess) \
      return BSA_ERR_CUDA;                                                                        \
    cudaEvent_t e2;                                                                               \
    const int w2 = timed_begin(BSA_TIMED_BWD_DQ, s, &e2);                                         \
    k2<<<grid, kBwdThreads, s2, s>>>(maps[0], maps[5], maps[1], maps[2], maps[3], maps[4], c);   \
    timed_end(w2, s, e2);                                                                         \
    if (cudaGetLastError() != cudaSuccess) return BSA_ERR_CUDA;                                   \
  } while (0)
  if (g.D == 128) BSA_LAUNCH_BWD(128);
  else BSA_LAUNCH_BWD(64);
#undef BSA_LAUNCH_BWD
  return BSA_OK;
}

}  // namespace bsa
