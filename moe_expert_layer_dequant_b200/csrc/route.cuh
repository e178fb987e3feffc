// Launch interface of the routing kernels (route.cu).
#pragma once
#include "common.cuh"

namespace moeffn {

constexpr int kMaxTopK = 16;
constexpr int kMaxExperts = 1024;

struct RouterArgs {
  const void* router;          // [E][H], fp32 or bf16
  bool router_f32;
  const uint16_t* w_sg;        // [H] bf16 shared-expert gate vector, or null
  const uint16_t* x;           // [M][H]
  int M, H, E;
  float* logits;               // [M][E]
  float* gate_logit;           // [M] (when w_sg != null)
};

struct RouteArgs {
  const float* logits;         // [M][E]
  int M, E, k;
  int* idx;                    // [M][k]
  float* w;                    // [M][k] fp16-rounded weights
  int* perm;                   // [M*k] or null (then nothing below is written)
  int* inv;                    // [M*k] position of pair p in perm, or null
  int* offsets;                // [E+1]
  int* union_list;             // [E] or null
  int* n_union;                // [1] or null
};

// xg[s][:] = x[perm[s] / topk][:] for the P = M*topk pair slots (bf16 rows of H).
struct GatherArgs {
  const uint16_t* x;
  const int* perm;
  int topk, H, P;
  uint16_t* xg;
};

cudaError_t launch_router_logits(const RouterArgs& a, cudaStream_t s);
cudaError_t launch_gather_rows(const GatherArgs& a, cudaStream_t s);
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);

}  // namespace moeffn
