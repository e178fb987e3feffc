// Launch interface of the tcgen05 quantized GEMM (gemm_tc.cu).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace moeffn {

enum : int { TC_GATEUP = 2, TC_DOWN = 1 };

// Tensor maps of one quantized matrix for the GEMM: codes (uint8, 128-byte
// swizzled boxes of [tile rows][128 bytes]), INT4 scales and mins (u16 boxes
// of [tile rows][8 groups]). The box height is the tile's weight rows per
// matrix: F for gate and up (GATEUP), R for down.
struct TcMaps {
  CUtensorMap codes, scale, mn;
};

struct TcGemmArgs {
  CUtensorMap xmap;            // A operand rows (dense / routed jobs): bf16 [rows][K], boxes [128][64]
  CUtensorMap xmap_s;          // A operand rows of the shared job
  TcMaps w0, w1;               // dense mode: gate, up (GATEUP) or down (w0)
  const TcMaps* tab0;          // grouped mode: per expert [E]
  const TcMaps* tab1;
  TcMaps s0, s1;               // shared expert
  const __half* rscale0;       // INT8 dense: per-row scales of w0 / w1
  const __half* rscale1;
  int fmt, act, mode;
  int mt;                      // 128-row token tiles per CTA (1 or 2)
  int tile, tile_s;            // features per tile (GATEUP, <= 128) or output rows (DOWN, <= 256)
  int N, K, Ns, Ks;            // dense / routed and shared shapes (rows, reduction)
  int M;
  const int* offsets;          // null: dense mode
  const int* union_list;
  const int* n_union;
  int routed_jobs;
  int slots;                   // slot count of the outputs (dense: M, grouped: M*topk)
  uint16_t* out_act;           // GATEUP: [slots][N] bf16
  uint16_t* out_act_s;         // [M][Ns]
  float* out_d;                // DOWN: [splits][slots][N] fp32
  float* out_d_s;              // [splits][M][N]
  int ks_len;                  // K per split (multiple of the weight stage K)
  int token_tiles;             // grid.y = token_tiles * splits
};

// K covered by one weight stage: 256 codes (INT4) or 128 (INT8).
inline int tc_k_tile(int fmt) { return fmt == FMT_INT4_G32 ? 256 : 128; }
// Features per GATEUP tile for an intermediate size I, rows per DOWN tile for
// an output size H.
int tc_gateup_feat(int I);
int tc_down_rows(int H);
// Token tiles per CTA for an expected token count per weight matrix, and the
// token rows one CTA covers.
int tc_mt_for(int tokens);
int tc_tokens_per_cta(int mt);

cudaError_t encode_tc_weight_maps(TcMaps* m, int fmt, const QW& w, int N, int K, int box_rows);
cudaError_t encode_tc_x_map(CUtensorMap* m, const uint16_t* x, int rows, int K);
cudaError_t launch_tc_gemm(const TcGemmArgs& a, int row_tiles, int splits, int jobs, cudaStream_t s);
unsigned int tc_gemm_fault_flags(bool clear);

}  // namespace moeffn
