// Launch interface of the tcgen05 quantized GEMM (gemm_tc.cu).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace moeffn {

enum : int { TC_GATEUP = 2, TC_DOWN = 1 };

// Weight rows of one MMA A tile, and token rows (MMA N) one CTA covers at most.
constexpr int kTcRowsA = 128;
constexpr int kTcMaxTok = 192;

// Tensor maps of one quantized matrix for the GEMM, boxes of kTcRowsA rows:
// codes (uint8, 128-byte swizzled [128 rows][128 bytes]; Q4_K: unswizzled
// [128 rows][one 144-byte block]), INT4 scales and mins (u16 [128 rows][8 groups]).
struct TcMaps {
  CUtensorMap codes, scale, mn;
};

struct TcGemmArgs {
  CUtensorMap xmap;            // B operand rows (dense / routed jobs): bf16 [rows][K], boxes [ntile][64]
  CUtensorMap xmap_s;          // B operand rows of the shared job
  TcMaps w0, w1;               // dense mode: gate, up (GATEUP) or down (w0)
  const TcMaps* tab0;          // grouped mode: per expert [E]
  const TcMaps* tab1;
  TcMaps s0, s1;               // shared expert
  const __half* rscale0;       // INT8 dense: per-row scales of w0 / w1
  const __half* rscale1;
  int fmt, act, mode;
  int ntile;                   // token rows per CTA tile (multiple of 16, <= kTcMaxTok; the maps' box height)
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
  int token_tiles;             // grid.z = token_tiles * splits (token tile major)
};

// K covered by one weight stage: 256 codes (INT4, Q4_K) or 128 (INT8).
inline int tc_k_tile(int fmt) { return fmt == FMT_INT8_ROW ? 128 : 256; }
// Output features per CTA (GATEUP: 128 gate rows and the same 128 up rows) and
// output rows per CTA (DOWN: two tiles of 128).
constexpr int kTcGateUpFeat = kTcRowsA;
constexpr int kTcDownRows = 2 * kTcRowsA;
// Token rows per CTA tile for `tokens` rows in a job: the fewest tiles of at
// most kTcMaxTok, balanced, rounded up to the MMA's N granule of 16.
int tc_ntile_for(int tokens);

cudaError_t encode_tc_weight_maps(TcMaps* m, int fmt, const QW& w, int N, int K);
cudaError_t encode_tc_x_map(CUtensorMap* m, const uint16_t* x, int rows, int K, int ntile);
cudaError_t launch_tc_gemm(const TcGemmArgs& a, int row_tiles, int splits, int jobs, cudaStream_t s);
unsigned int tc_gemm_fault_flags(bool clear);

}  // namespace moeffn
