// Launch accounting and optional per-kernel timing.
//
// Every kernel launch made by the library goes through a ProfileScope.  The
// scope always counts the launch (per kernel kind); when timing is enabled
// it also records a pair of CUDA events around the launch on the launching
// stream, so ft_profile_read can report the device time of each kind.
// Timing is skipped while the stream is being captured into a graph.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "ftmoe.h"

namespace ftmoe {

struct Profiler {
  std::atomic<long long> launches[FT_KERNEL_KINDS];
  std::atomic<int> enabled{0};
  std::mutex mu;
  struct Rec { int kind; cudaEvent_t a, b; };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> spare;
  Profiler() { for (auto& l : launches) l = 0; }

  cudaEvent_t take() {
    if (!spare.empty()) { cudaEvent_t e = spare.back(); spare.pop_back(); return e; }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

static Profiler& profiler() {
  static Profiler* p = new Profiler();   // never destroyed: events may outlive static teardown
  return *p;
}

class ProfileScope {
 public:
  ProfileScope(int kind, cudaStream_t s) : kind_(kind), s_(s) {
    Profiler& P = profiler();
    P.launches[kind].fetch_add(1, std::memory_order_relaxed);
    if (!P.enabled.load(std::memory_order_relaxed)) return;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return;
    std::lock_guard<std::mutex> g(P.mu);
    a_ = P.take();
    b_ = P.take();
    if (a_ && b_) cudaEventRecord(a_, s_);
  }
  ~ProfileScope() {
    if (!a_ || !b_) return;
    Profiler& P = profiler();
    std::lock_guard<std::mutex> g(P.mu);
    cudaEventRecord(b_, s_);
    P.pending.push_back({kind_, a_, b_});
  }
  ProfileScope(const ProfileScope&) = delete;
  ProfileScope& operator=(const ProfileScope&) = delete;

 private:
  int kind_;
  cudaStream_t s_;
  cudaEvent_t a_ = nullptr, b_ = nullptr;
};

}  // namespace ftmoe
