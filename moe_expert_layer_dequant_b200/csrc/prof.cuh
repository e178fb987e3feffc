// Optional per-launch timing of the library's kernels with CUDA events.
#pragma once
#include <cuda_runtime.h>

namespace moeffn {

bool prof_enabled();
void prof_begin(const char* name, cudaStream_t s);
void prof_end(cudaStream_t s);

// Brackets one kernel launch with events when profiling is on.
struct ProfScope {
  cudaStream_t s;
  bool on;
  ProfScope(const char* name, cudaStream_t st) : s(st), on(prof_enabled()) {
    if (on) prof_begin(name, s);
  }
  ~ProfScope() {
    if (on) prof_end(s);
  }
};

}  // namespace moeffn
