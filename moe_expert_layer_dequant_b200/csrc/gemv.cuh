// Launch interface of the decode GEMV kernels (gemv.cu).
#pragma once
#include "common.cuh"

namespace moeffn {

// Fused gate/up projection + gated activation: out = bf16(act(Wg x) * (Wu x)).
struct GateUpArgs {
  int fmt, act;
  int K;                       // input width (hidden size)
  QW g, u;                     // dense mode matrices
  const QW* g_tab;             // grouped mode: per-expert tables (device)
  const QW* u_tab;
  int N;                       // rows of the dense / routed gate and up matrices
  QW sg, su;                   // shared expert (grouped mode), Ns = 0 if none
  int Ns;
  const uint16_t* x;           // [M][K] bf16
  int M, topk;
  const int* perm;             // null: dense mode
  const int* offsets;
  const int* union_list;
  const int* n_union;
  int routed_jobs;             // grid.y slots given to routed jobs
  uint16_t* out;               // dense: [M][N]; grouped: [M*topk][N] slot order
  uint16_t* out_s;             // shared: [M][Ns]
  int rows_per_cta;
  int stage_tokens;            // token rows staged in shared memory at once
};

// Down projection, split along K: d[split][slot][n] = sum over the split's K range.
struct DownArgs {
  int fmt;
  int K, N;                    // routed / dense: K = intermediate width, N = hidden rows
  QW w;                        // dense mode matrix
  const QW* tab;               // grouped mode: per-expert table (device)
  QW ws;                       // shared expert down (K = Ks)
  int Ks;
  const uint16_t* in;          // [slots][K] bf16 activations (slot order)
  const uint16_t* in_s;        // [M][Ks]
  int M, slots;                // slots = M (dense) or M*topk (grouped)
  const int* offsets;          // null: dense mode
  const int* union_list;
  const int* n_union;
  int routed_jobs;
  float* d;                    // [splits][slots][N]
  float* d_s;                  // [splits][M][N]
  int ks_len;                  // K elements per split (multiple of 32)
  int rows_per_cta;
  int stage_tokens;
};

size_t gemv_stage_bytes(int fmt, int klen, int tokens);
cudaError_t launch_gateup(const GateUpArgs& a, int grid_x, int jobs, int mt, cudaStream_t s);
cudaError_t launch_down(const DownArgs& a, int grid_x, int splits, int jobs, int mt, cudaStream_t s);

}  // namespace moeffn
