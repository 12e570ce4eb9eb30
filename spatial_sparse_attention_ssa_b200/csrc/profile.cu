// Per-kernel timing and launch counting for libssa (tracing subsystem).
//
// Every kernel launch of the library goes through prof_begin / prof_end (see
// SSA_LAUNCH in common.cuh).  Counting is always on; timing is on between
// ssa_profile_enable(1) and ssa_profile_enable(0): a CUDA event pair is recorded
// on the launching stream around each launch, and ssa_profile_read aggregates
// the elapsed times per kernel name.
#include <mutex>
#include <string.h>
#include <string>
#include <vector>

#include "common.cuh"

namespace ssa {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_enabled = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;
unsigned long long g_launches = 0;
thread_local const char* t_name = nullptr;
thread_local cudaEvent_t t_begin = nullptr;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

void prof_begin(const char* name, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  ++g_launches;
  if (!g_enabled) return;
  t_name = name;
  t_begin = take_event();
  cudaEventRecord(t_begin, st);
}

void prof_end(cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_enabled || !t_begin) return;
  cudaEvent_t e = take_event();
  cudaEventRecord(e, st);
  g_recs.push_back({t_name, t_begin, e});
  t_begin = nullptr;
}

}  // namespace ssa

extern "C" {

SSA_API void ssa_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(ssa::g_mu);
  ssa::g_enabled = on != 0;
}

SSA_API uint64_t ssa_launch_count(void) {
  std::lock_guard<std::mutex> lk(ssa::g_mu);
  return ssa::g_launches;
}

SSA_API int32_t ssa_profile_read(char* names, int32_t name_len, float* total_ms, int32_t* launches,
                                 int32_t max_entries) {
  std::lock_guard<std::mutex> lk(ssa::g_mu);
  std::vector<std::string> keys;
  std::vector<double> tot;
  std::vector<int> cnt;
  for (auto& r : ssa::g_recs) {
    cudaEventSynchronize(r.b);
    float ms = 0.f;
    cudaEventElapsedTime(&ms, r.a, r.b);
    size_t i = 0;
    for (; i < keys.size(); ++i)
      if (keys[i] == r.name) break;
    if (i == keys.size()) {
      keys.push_back(r.name);
      tot.push_back(0.0);
      cnt.push_back(0);
    }
    tot[i] += ms;
    cnt[i] += 1;
    ssa::g_pool.push_back(r.a);
    ssa::g_pool.push_back(r.b);
  }
  ssa::g_recs.clear();
  const int n = (int)keys.size() < max_entries ? (int)keys.size() : max_entries;
  for (int i = 0; i < n; ++i) {
    if (names && name_len > 0) {
      strncpy(names + (size_t)i * name_len, keys[i].c_str(), name_len - 1);
      names[(size_t)i * name_len + name_len - 1] = 0;
    }
    if (total_ms) total_ms[i] = (float)tot[i];
    if (launches) launches[i] = cnt[i];
  }
  return (int32_t)keys.size();
}

}  // extern "C"
