// timing.cu -- optional per-kernel CUDA-event timing (a measurement aid, off by default).
// While enabled, every kernel launch of the library is bracketed by two events on its
// stream; zipnn_timing_collect waits for them and reports the summed durations.
#include <mutex>
#include <vector>

#include "zipnn.h"
#include "launch.h"

namespace zipnn {
namespace {

const char* const kNames[kNumKernelIds] = {"split_hist", "code_build", "layout_scan", "encode",
                                           "decode_merge", "code_lengths", "plan", "shard_tables",
                                           "pack_hist", "pack_encode"};

struct Pending {
  int id;
  cudaEvent_t start, stop;
};

struct Timing {
  std::mutex mu;
  bool enabled = false;
  std::vector<cudaEvent_t> pool;
  std::vector<Pending> pending;
  double ms[kNumKernelIds] = {0};
  uint64_t launches[kNumKernelIds] = {0};
};

Timing& timing() {
  static Timing t;
  return t;
}

cudaEvent_t take_event(Timing& t) {
  if (!t.pool.empty()) {
    cudaEvent_t e = t.pool.back();
    t.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

TimedLaunch::TimedLaunch(int id, cudaStream_t st) : id_(id), st_(st) {
  Timing& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  if (!t.enabled) return;
  start_ = take_event(t);
  stop_ = take_event(t);
  if (start_ && stop_) cudaEventRecord(start_, st_);
}

TimedLaunch::~TimedLaunch() {
  if (!start_ || !stop_) return;
  Timing& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  cudaEventRecord(stop_, st_);
  t.pending.push_back({id_, start_, stop_});
}

}  // namespace zipnn

using namespace zipnn;

extern "C" {

zipnn_status zipnn_timing_enable(int enable) {
  Timing& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  t.enabled = enable != 0;
  return ZIPNN_OK;
}

zipnn_status zipnn_timing_collect(double* ms, uint64_t* launches, uint32_t count) {
  Timing& t = timing();
  std::lock_guard<std::mutex> g(t.mu);
  zipnn_status st = ZIPNN_OK;
  for (const Pending& p : t.pending) {
    float f = 0.f;
    if (cudaEventSynchronize(p.stop) != cudaSuccess || cudaEventElapsedTime(&f, p.start, p.stop) != cudaSuccess) {
      st = ZIPNN_ERR_CUDA;
    } else {
      t.ms[p.id] += f;
      t.launches[p.id] += 1;
    }
    t.pool.push_back(p.start);
    t.pool.push_back(p.stop);
  }
  t.pending.clear();
  for (uint32_t i = 0; i < count && i < (uint32_t)kNumKernelIds; i++) {
    if (ms) ms[i] = t.ms[i];
    if (launches) launches[i] = t.launches[i];
  }
  for (int i = 0; i < kNumKernelIds; i++) {
    t.ms[i] = 0;
    t.launches[i] = 0;
  }
  return st;
}

uint32_t zipnn_kernel_count(void) { return (uint32_t)kNumKernelIds; }

const char* zipnn_kernel_name(uint32_t id) { return id < (uint32_t)kNumKernelIds ? kNames[id] : "unknown"; }

}  // extern "C"
