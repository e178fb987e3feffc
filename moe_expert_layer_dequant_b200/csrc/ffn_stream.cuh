// Launch interface of the single-stream dense FFN for one or two token rows
// (ffn_stream.cu).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "gemv_tma.cuh"

namespace moeffn {

enum : int { STREAM_RESIDUAL = 0, STREAM_RMSNORM = 1 };

struct FfnStreamArgs {
  QWMaps maps_a[2];            // gate, up: boxes of [8 rows][box_a codes]
  QWMaps map_down;             // down: boxes of [4 rows][box_b codes]
  const __half* rs_gate;       // INT8 row scales
  const __half* rs_up;
  const __half* rs_down;
  int H, I, M, act;
  float eps;
  const uint16_t* x;           // [M][H]
  uint16_t* res;               // residual mode: [M][H], updated in place
  uint16_t* out;               // RMSNorm mode: [M][H]
  const uint16_t* norm_w;      // [H]
  uint16_t* hbuf;              // [M][I] gated activations (workspace)
  float* ybuf;                 // [M][H] pre-norm outputs (workspace, RMSNorm mode)
  int kc_a, box_a, kc_b, box_b;   // K codes per stage and per box, phases A and B
  int blocks_a, blocks_b;      // row blocks of the two phases
  int stages, stage_bytes, stage_x_bytes;
  size_t smem;
};

// Fills the geometry of a (H, I, M) problem; false when the shapes do not fit
// (then the GEMV launches are used).
bool ffn_stream_plan(FfnStreamArgs* a, int fmt, int H, int I, int M);
cudaError_t ffn_stream_encode(FfnStreamArgs* a, int fmt, const QW& gate, const QW& up, const QW& down);
cudaError_t launch_ffn_stream(const FfnStreamArgs& a, int fmt, int mode, cudaStream_t s);
unsigned int ffn_stream_fault_flags(bool clear);

}  // namespace moeffn
