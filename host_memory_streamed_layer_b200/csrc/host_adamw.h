// Host-side optimizer and worker pool.
//
// MegaTrain keeps the fp32 master weights and both Adam moments in host memory
// and updates them on the CPU (intelligentliving.co, "Checkpointing, Manual
// Gradients, and CPU-Side Optimizer Steps"; MegaTrain abstract). The update is
// AdamW (Kingma & Ba, "Adam: A Method for Stochastic Optimization", with
// decoupled weight decay), fused with the round-to-nearest-even bf16 copy that
// the next step streams to the GPU.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <condition_variable>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

namespace mt {

struct AdamHyper {
  float lr, beta1, beta2, eps, wd;
};

// One AdamW step over n elements, in place:
//   p <- p (1 - lr wd); m <- b1 m + (1 - b1) g; v <- b2 v + (1 - b2) g^2;
//   p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// and pb[i] <- bf16(p[i]) (round to nearest even) when pb is not null.
// g == nullptr means a zero gradient (nothing is read).
void adamw_chunk(float* p, const float* g, float* m, float* v, uint16_t* pb, size_t n, const AdamHyper& h, int t);

// The same step with a bf16 gradient (bit patterns, widened exactly to fp32).
void adamw_chunk_bf16g(float* p, const uint16_t* g, float* m, float* v, uint16_t* pb, size_t n, const AdamHyper& h,
                       int t);

// Round-to-nearest-even fp32 -> bf16 over n elements (NaN stays NaN).
void bf16_round_chunk(const float* x, uint16_t* out, size_t n);
uint16_t bf16_rne(float x);

// True when the AVX-512 path is in use on this CPU.
bool adamw_uses_avx512();

// Fixed set of worker threads; run() executes fn(i) for i in [0, n) on the
// workers and the calling thread and returns when every call has finished.
class ThreadPool {
 public:
  explicit ThreadPool(int workers);
  ~ThreadPool();
  void run(int n, const std::function<void(int)>& fn);
  int size() const { return (int)workers_.size() + 1; }

 private:
  void loop();
  std::vector<std::thread> workers_;
  std::mutex mu_;
  std::condition_variable cv_, done_cv_;
  const std::function<void(int)>* fn_ = nullptr;
  int n_ = 0;
  std::atomic<int> next_{0};
  int finished_ = 0;
  int active_ = 0;
  uint64_t gen_ = 0;
  bool stop_ = false;
};

// Splits [0, n) into contiguous chunks (multiples of 64 elements) and runs
// body(begin, end) over the pool.
void parallel_ranges(ThreadPool& pool, size_t n, const std::function<void(size_t, size_t)>& body);

}  // namespace mt
