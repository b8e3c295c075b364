// Per-kernel tracing: when enabled, every launch the library makes is
// bracketed by a pair of CUDA events on its stream; hstu_trace_read sums the
// device time per kernel name.  Disabled (the default) it costs one branch.
#include <mutex>
#include <string.h>
#include <string>
#include <vector>

#include "common.cuh"
#include "trace.cuh"

namespace hstu {
namespace {
struct Rec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t get_event() {
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

bool trace_on() { return g_on; }

int trace_begin(const char* name, cudaStream_t st) {
  if (!g_on) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  Rec r{name, get_event(), get_event()};
  if (!r.a || !r.b) return -1;
  cudaEventRecord(r.a, st);
  g_recs.push_back(r);
  return (int)g_recs.size() - 1;
}

void trace_end(int h, cudaStream_t st) {
  if (h < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (h < (int)g_recs.size()) cudaEventRecord(g_recs[h].b, st);
}

}  // namespace hstu

using namespace hstu;

extern "C" {

int hstu_trace_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& r : g_recs) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  g_on = enable != 0;
  return HSTU_OK;
}

int hstu_trace_read(int32_t max_kernels, char* names, int32_t* counts, double* total_ms, int32_t* num_kernels) {
  if (max_kernels < 0 || !num_kernels || (max_kernels > 0 && (!names || !counts || !total_ms)))
    return HSTU_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  std::vector<std::string> keys;
  std::vector<int32_t> cnt;
  std::vector<double> ms;
  for (auto& r : g_recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return HSTU_ERR_CUDA;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return HSTU_ERR_CUDA;
    size_t k = 0;
    for (; k < keys.size(); ++k)
      if (keys[k] == r.name) break;
    if (k == keys.size()) {
      keys.push_back(r.name);
      cnt.push_back(0);
      ms.push_back(0.0);
    }
    cnt[k] += 1;
    ms[k] += t;
  }
  *num_kernels = (int32_t)keys.size();
  for (size_t k = 0; k < keys.size() && (int)k < max_kernels; ++k) {
    strncpy(names + 32 * k, keys[k].c_str(), 31);
    names[32 * k + 31] = 0;
    counts[k] = cnt[k];
    total_ms[k] = ms[k];
  }
  return HSTU_OK;
}

}  // extern "C"
