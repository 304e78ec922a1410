// Host-side launch accounting for the library's kernels.
//
// Every kernel launch of the library is counted.  When profiling is enabled, each launch is
// also bracketed by two CUDA events recorded on the launching stream.  dp_profiling_collect
// then turns them into per-kind device time.  Events are stream-ordered markers: they do not
// serialise other streams or change what the kernels do.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

namespace dpclip {

enum KernelKind : int {
  kKindNoise = 0,
  kKindProjection,
  kKindPhilox,
  kKindScale,
  kKindFinalize,
  kKindF32Norm,
  kKindF32ClipSum,
  kKindF32Project,
  kKindClipSum,       // tcgen05 clipped sum + noise epilogue
  kKindExplicitNorm,  // tcgen05 per-sample G_i tiles, squared on chip
  kKindGhostNorm,     // tcgen05 Gram tiles of X_i and dY_i
  kKindProject,       // tcgen05 Z = dY P
  kKindExplicitStore, // tcgen05 per-sample G_i tiles, squared on chip and stored in bf16
  kKindReduce,        // sum_i c_i G_i over the stored tiles + noise
  kKindAdam,          // projected Adam moments and update in r-space
  kKindAxpy,          // tcgen05 W += alpha U P^T
  kKindGhostShared,   // tcgen05 one X Gram shared by the dY Grams of up to three linears
  kKindCombine,       // the split partials of clipped sums split over K, added in split order
  kNumKinds
};

inline const char* kernel_kind_name(int k) {
  static const char* names[kNumKinds] = {
      "noise_add",  "projection",   "philox_blocks", "scale_rows_bf16", "finalize_norms",
      "f32_norm",   "f32_clipsum",  "f32_project",   "umma_clipsum",    "umma_explicit_norm",
      "umma_ghost_norm", "umma_project", "umma_explicit_store", "clip_reduce", "adam_rspace",
      "umma_axpy", "umma_ghost_shared", "split_combine"};
  return (k >= 0 && k < kNumKinds) ? names[k] : "";
}

struct LaunchProfiler {
  struct Rec {
    int kind;
    cudaEvent_t a, b;
  };
  std::mutex mu;
  bool enabled = false;
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  std::atomic<long long> launches{0};
  std::atomic<long long> per_kind[kNumKinds] = {};

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  void give(cudaEvent_t e) {
    if (e) pool.push_back(e);
  }
};

inline LaunchProfiler& profiler() {
  static LaunchProfiler p;
  return p;
}

// Brackets one launch: construct before the <<<>>> launch, destroy after it.
class LaunchScope {
 public:
  LaunchScope(int kind, cudaStream_t stream) : kind_(kind), stream_(stream) {
    LaunchProfiler& p = profiler();
    p.launches.fetch_add(1, std::memory_order_relaxed);
    p.per_kind[kind].fetch_add(1, std::memory_order_relaxed);
    std::lock_guard<std::mutex> g(p.mu);
    if (p.enabled) {
      a_ = p.take();
      if (a_) cudaEventRecord(a_, stream_);
    }
  }
  ~LaunchScope() {
    if (!a_) return;
    LaunchProfiler& p = profiler();
    std::lock_guard<std::mutex> g(p.mu);
    cudaEvent_t b = p.take();
    if (!b) {
      p.give(a_);
      return;
    }
    cudaEventRecord(b, stream_);
    p.recs.push_back({kind_, a_, b});
  }

 private:
  int kind_;
  cudaStream_t stream_;
  cudaEvent_t a_ = nullptr;
};

}  // namespace dpclip
