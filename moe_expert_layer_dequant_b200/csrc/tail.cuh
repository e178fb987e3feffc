// Launch interface of the tail kernels (tail.cu).
#pragma once
#include "common.cuh"

namespace moeffn {

enum : int { TAIL_RESIDUAL = 0, TAIL_RMSNORM = 1, TAIL_MOE = 2, TAIL_MOE_GEMMA = 3 };

struct TailArgs {
  int mode;
  int M, N;                    // token rows, hidden size
  const float* d;              // [splits][slots][N] partial down outputs
  int splits, slots;
  const float* d_s;            // [splits_s][M][N] shared-expert down partials, or null
  int splits_s;
  const float* gate_logit;     // [M] shared-expert gate logits
  const float* w;              // [M][k] routing weights
  const int* inv;              // [M*k] slot of pair p
  int k;
  uint16_t* res;               // [M][N] residual stream, updated in place
  uint16_t* h1;                // [M][N] RMSNorm output
  const uint16_t* norm_w;      // [N] (RMSNORM: the branch's norm; MOE_GEMMA: the shared branch's post-norm)
  float eps;
};

cudaError_t launch_tail(const TailArgs& a, cudaStream_t s);

}  // namespace moeffn
