// Per-launch event timing (moeffn_profile_enable / moeffn_profile_read).
// Off by default; while on, each kernel launch of the library is bracketed by
// two events recorded on the launch's stream, so the device time of every
// launch can be read back per kernel name.
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/moeffn.h"
#include "prof.cuh"

namespace moeffn {
int api_fail(int code, const char* msg);

namespace {
struct Rec {
  const char* name;
  cudaEvent_t start, stop;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;       // recorded since the last read
std::vector<cudaEvent_t> g_pool;
size_t g_open = 0;             // index of the record awaiting its stop event

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

bool prof_enabled() { return g_on; }

void prof_begin(const char* name, cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  Rec r{name, take_event(), take_event()};
  cudaEventRecord(r.start, s);
  g_recs.push_back(r);
  g_open = g_recs.size() - 1;
}

void prof_end(cudaStream_t s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_open < g_recs.size()) cudaEventRecord(g_recs[g_open].stop, s);
}

}  // namespace moeffn

using namespace moeffn;

extern "C" {

int moeffn_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = on != 0;
  return MOEFFN_OK;
}

int moeffn_profile_read(char* names, int names_len, int* counts, float* total_ms, int max_kernels, int* n_kernels) {
  std::lock_guard<std::mutex> lk(g_mu);
  std::vector<std::string> uniq;
  std::vector<int> cnt;
  std::vector<double> ms;
  cudaError_t err = cudaSuccess;
  for (const Rec& r : g_recs) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.stop);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.start, r.stop);
    if (e != cudaSuccess) err = e;
    size_t i = 0;
    while (i < uniq.size() && uniq[i] != r.name) ++i;
    if (i == uniq.size()) {
      uniq.emplace_back(r.name);
      cnt.push_back(0);
      ms.push_back(0.0);
    }
    cnt[i] += 1;
    ms[i] += t;
    g_pool.push_back(r.start);
    g_pool.push_back(r.stop);
  }
  g_recs.clear();
  if (err != cudaSuccess) return api_fail(MOEFFN_ERR_CUDA, cudaGetErrorString(err));
  if (n_kernels) *n_kernels = (int)uniq.size();
  std::string joined;
  for (size_t i = 0; i < uniq.size() && (int)i < max_kernels; ++i) {
    if (counts) counts[i] = cnt[i];
    if (total_ms) total_ms[i] = (float)ms[i];
    joined += uniq[i];
    joined += '\n';
  }
  if (names && names_len > 0) {
    strncpy(names, joined.c_str(), names_len - 1);
    names[names_len - 1] = '\0';
  }
  return MOEFFN_OK;
}

}  // extern "C"
