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
  // Input norm folded in: x is the residual; the logits use m = rms_norm(x,
  // norm_w), which the (token, 0) CTAs also write to m_out [M][H]. Null: x is m.
  const uint16_t* norm_w;
  float eps;
  uint16_t* m_out;
  int* route_cnt;              // zeroed here for the top-k kernel that follows, or null
};

// m = rms_norm(x, w) row by row into m [M][H] (one CTA per row).
struct PrenormArgs {
  const uint16_t* x;
  const uint16_t* w;
  float eps;
  int M, H;
  uint16_t* m;
};
cudaError_t launch_prenorm_rows(const PrenormArgs& a, cudaStream_t s);

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
  const float* scale;          // [E] per-expert scale of the routing weights, or null (ones)
  int* counter;                // [1] arrival counter of the top-k CTAs, zero on entry (with perm)
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
