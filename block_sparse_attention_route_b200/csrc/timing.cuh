// timing.cuh -- opt-in CUDA-event timing of the attention kernels (bsa_kernel_timing).
//
// While enabled, each attention launch is bracketed by two events recorded on its own
// stream; bsa_kernel_times() sums the pairs per kernel.  Host-only bookkeeping: nothing here
// runs on the device, and with timing off (the default) a launch pays one atomic load.
#pragma once
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include <cuda_runtime.h>

namespace bsa {

constexpr int kNumTimed = 3;  // forward, backward dK/dV, backward dQ (BSA_TIMED_* order)

struct KernelTimer {
  std::atomic<int> on{0};
  std::mutex mu;
  std::vector<std::pair<cudaEvent_t, cudaEvent_t>> pending[kNumTimed];
  std::vector<cudaEvent_t> pool;

  cudaEvent_t take() {  // called with mu held
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

inline KernelTimer& kernel_timer() {
  static KernelTimer t;
  return t;
}

// Records the start event of kernel `which` on `s` when timing is on; returns the pair slot
// to close with timed_end (or -1).
inline int timed_begin(int which, cudaStream_t s, cudaEvent_t* start) {
  KernelTimer& t = kernel_timer();
  *start = nullptr;
  if (!t.on.load(std::memory_order_relaxed)) return -1;
  std::lock_guard<std::mutex> lk(t.mu);
  *start = t.take();
  if (*start == nullptr || cudaEventRecord(*start, s) != cudaSuccess) return -1;
  return which;
}
inline void timed_end(int which, cudaStream_t s, cudaEvent_t start) {
  if (which < 0 || start == nullptr) return;
  KernelTimer& t = kernel_timer();
  std::lock_guard<std::mutex> lk(t.mu);
  cudaEvent_t stop = t.take();
  if (stop == nullptr || cudaEventRecord(stop, s) != cudaSuccess) {
    t.pool.push_back(start);
    return;
  }
  t.pending[which].emplace_back(start, stop);
}

}  // namespace bsa
