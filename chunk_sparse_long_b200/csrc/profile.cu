// Per-kernel timing with CUDA events (hils_profile_* in include/hils.h).
//
// When enabled, every launcher brackets each kernel it enqueues with a pair of
// events recorded on the call's stream.  hils_profile_read() waits for the
// recorded events, folds them into per-phase totals and recycles them.  The
// events come from a small pool that grows on demand and is reused; no device
// memory is involved.  Not thread-safe: meant for a single benchmarking thread.
#include <cstring>
#include <string>
#include <vector>

#include "hils_common.cuh"

namespace hils {
namespace {

struct Record {
  const char* phase;
  cudaEvent_t start, stop;
};

struct Profiler {
  bool on = false;
  std::vector<cudaEvent_t> pool;
  std::vector<Record> pending;
  std::vector<std::string> names;
  std::vector<double> total_ms;
  std::vector<long long> launches;

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
};

Profiler& prof() {
  static Profiler p;
  return p;
}

}  // namespace

ProfileScope::ProfileScope(const char* phase, cudaStream_t s) : phase_(phase), stream_(s) {
  Profiler& p = prof();
  if (!p.on) return;
  start_ = p.take();
  if (start_) cudaEventRecord((cudaEvent_t)start_, s);
}

ProfileScope::~ProfileScope() {
  Profiler& p = prof();
  if (!p.on || !start_) return;
  cudaEvent_t stop = p.take();
  if (!stop) return;
  cudaEventRecord(stop, stream_);
  p.pending.push_back({phase_, (cudaEvent_t)start_, stop});
}

}  // namespace hils

extern "C" {

int hils_profile_enable(int on) {
  hils::prof().on = on != 0;
  return HILS_OK;
}

int hils_profile_collect(void) {
  hils::Profiler& p = hils::prof();
  for (auto& r : p.pending) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) return HILS_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) return HILS_ERR_CUDA;
    size_t i = 0;
    while (i < p.names.size() && p.names[i] != r.phase) ++i;
    if (i == p.names.size()) {
      p.names.emplace_back(r.phase);
      p.total_ms.push_back(0.0);
      p.launches.push_back(0);
    }
    p.total_ms[i] += ms;
    p.launches[i] += 1;
    p.pool.push_back(r.start);
    p.pool.push_back(r.stop);
  }
  p.pending.clear();
  return HILS_OK;
}

int hils_profile_read(int i, const char** name, double* total_ms, long long* launches) {
  hils::Profiler& p = hils::prof();
  if (i < 0 || i >= (int)p.names.size()) return HILS_ERR_INVALID_ARG;
  if (name) *name = p.names[i].c_str();
  if (total_ms) *total_ms = p.total_ms[i];
  if (launches) *launches = p.launches[i];
  return HILS_OK;
}

int hils_profile_reset(void) {
  hils::Profiler& p = hils::prof();
  hils_profile_collect();
  p.names.clear();
  p.total_ms.clear();
  p.launches.clear();
  return HILS_OK;
}

}  // extern "C"
