#include <atomic>
#include <mutex>
#include <vector>

#include "dash_b200.h"
#include "profile.cuh"

namespace dash {

int gemm_wide_regs();  // gemm_wide.cu
namespace {

struct Rec {
  int stage;
  double flops;
  cudaEvent_t start, stop;
};

struct Prof {
  std::mutex mu;
  std::atomic<bool> on{false};
  std::atomic<long long> launches{0};
  std::vector<Rec> recs;         // recorded pairs since the last reset
  std::vector<cudaEvent_t> pool;  // spare events
  long long dropped = 0;
};

Prof& prof() {
  static Prof* p = new Prof();  // never destroyed: events may outlive static destruction order
  return *p;
}

constexpr size_t kMaxRecs = 1 << 16;

cudaEvent_t take_event(Prof& p) {
  if (!p.pool.empty()) {
    cudaEvent_t e = p.pool.back();
    p.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

bool prof_on() { return prof().on.load(std::memory_order_relaxed); }

void prof_count_launch(int n) { prof().launches.fetch_add(n, std::memory_order_relaxed); }

int prof_begin(int stage, cudaStream_t st, double flops) {
  Prof& p = prof();
  if (!p.on.load(std::memory_order_relaxed)) return -1;
  std::lock_guard<std::mutex> lk(p.mu);
  if (p.recs.size() >= kMaxRecs) {
    ++p.dropped;
    return -1;
  }
  Rec r{stage, flops, take_event(p), take_event(p)};
  if (!r.start || !r.stop || cudaEventRecord(r.start, st) != cudaSuccess) {
    ++p.dropped;
    return -1;
  }
  p.recs.push_back(r);
  return static_cast<int>(p.recs.size()) - 1;
}

void prof_end(int slot, cudaStream_t st) {
  if (slot < 0) return;
  Prof& p = prof();
  std::lock_guard<std::mutex> lk(p.mu);
  if (slot < static_cast<int>(p.recs.size())) cudaEventRecord(p.recs[slot].stop, st);
}

}  // namespace dash

extern "C" {

SHAMPOO_API int shampoo_profile_enable(int enable) {
  dash::prof().on.store(enable != 0);
  return SHAMPOO_OK;
}

SHAMPOO_API int shampoo_profile_reset(void) {
  dash::Prof& p = dash::prof();
  std::lock_guard<std::mutex> lk(p.mu);
  for (auto& r : p.recs) {
    p.pool.push_back(r.start);
    p.pool.push_back(r.stop);
  }
  p.recs.clear();
  p.dropped = 0;
  p.launches.store(0);
  return SHAMPOO_OK;
}

SHAMPOO_API int shampoo_profile_read(double* out, int n) {
  if (!out || n < 3 * dash::kProfStages + 3) return SHAMPOO_EINVAL;
  dash::Prof& p = dash::prof();
  std::lock_guard<std::mutex> lk(p.mu);
  for (int i = 0; i < 3 * dash::kProfStages + 3; ++i) out[i] = 0.0;
  for (auto& r : p.recs) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return SHAMPOO_ECUDA;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return SHAMPOO_ECUDA;
    out[3 * r.stage] += ms;
    out[3 * r.stage + 1] += 1.0;
    out[3 * r.stage + 2] += r.flops;
  }
  out[3 * dash::kProfStages] = static_cast<double>(p.launches.load());
  out[3 * dash::kProfStages + 1] = static_cast<double>(p.dropped);
  out[3 * dash::kProfStages + 2] = static_cast<double>(dash::gemm_wide_regs());
  return SHAMPOO_OK;
}

}  // extern "C"
