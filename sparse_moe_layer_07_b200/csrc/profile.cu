// Phase timing of the training pair (moe_profile_phases / moe_profile_read):
// CUDA event pairs around kernels, recorded only while enabled, summed per
// phase on read.  Host code only; events are pooled and reused.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "internal.h"
#include "moe.h"

namespace moe {
namespace {

constexpr size_t kMaxPending = 65536;

struct Pending {
  int phase;
  cudaEvent_t a, b;
};

struct ProfileState {
  std::mutex mu;
  bool on = false;
  std::vector<Pending> pending;
  std::vector<cudaEvent_t> pool;
};

ProfileState& state() {
  static ProfileState* s = new ProfileState();  // never destroyed: events may outlive static teardown order
  return *s;
}

cudaEvent_t take_event(ProfileState& st) {
  if (!st.pool.empty()) {
    cudaEvent_t e = st.pool.back();
    st.pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return e;
}

}  // namespace

PhaseMark::PhaseMark(int phase, cudaStream_t s) : phase_(phase), s_(s) {
  ProfileState& st = state();
  std::lock_guard<std::mutex> lock(st.mu);
  if (!st.on || st.pending.size() >= kMaxPending) return;
  a_ = take_event(st);
  b_ = take_event(st);
  if (!a_ || !b_ || cudaEventRecord(a_, s_) != cudaSuccess) {
    (void)cudaGetLastError();
    if (a_) st.pool.push_back(a_);
    if (b_) st.pool.push_back(b_);
    a_ = b_ = nullptr;
  }
}

void PhaseMark::end() {
  if (!a_) return;
  ProfileState& st = state();
  std::lock_guard<std::mutex> lock(st.mu);
  if (cudaEventRecord(b_, s_) == cudaSuccess) {
    st.pending.push_back({phase_, a_, b_});
  } else {
    (void)cudaGetLastError();
    st.pool.push_back(a_);
    st.pool.push_back(b_);
  }
  a_ = b_ = nullptr;
}

}  // namespace moe

extern "C" {

moe_status_t moe_profile_phases(int32_t enable) {
  moe::ProfileState& st = moe::state();
  std::lock_guard<std::mutex> lock(st.mu);
  st.on = enable != 0;
  return MOE_OK;
}

moe_status_t moe_profile_read(float* ms, int32_t* calls, int32_t n) {
  if (n < 0) return MOE_ERR_INVALID_ARG;
  moe::ProfileState& st = moe::state();
  std::vector<moe::Pending> todo;
  {
    std::lock_guard<std::mutex> lock(st.mu);
    todo.swap(st.pending);
  }
  for (int32_t p = 0; p < n; ++p) {
    if (ms) ms[p] = 0.f;
    if (calls) calls[p] = 0;
  }
  bool ok = true;
  for (const moe::Pending& r : todo) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) {
      (void)cudaGetLastError();
      ok = false;
      continue;
    }
    if (r.phase >= 0 && r.phase < n) {
      if (ms) ms[r.phase] += t;
      if (calls) calls[r.phase] += 1;
    }
  }
  {
    std::lock_guard<std::mutex> lock(st.mu);
    for (const moe::Pending& r : todo) {
      st.pool.push_back(r.a);
      st.pool.push_back(r.b);
    }
  }
  return ok ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"
