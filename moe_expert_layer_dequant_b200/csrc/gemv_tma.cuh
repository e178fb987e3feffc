// Launch interface of the TMA-fed GEMV (gemv_tma.cu).
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace moeffn {

constexpr int kTmaConsumers = 8;  // consumer warps per group = rows per stage
// Consumer groups, taking stages in turn. Two: a stage of two matrices (gate
// and up) or of one matrix's row pairs (down) is twice the bytes of a single
// row set, and a third group (800 threads) would leave each thread too few
// registers for the two rows' accumulators.
constexpr int kTmaGroups = 2;
// Token rows whose input norm the GEMV's staging applies (more: a norm launch first).
constexpr int kGemvNormTokens = 8;
// Shared memory of the staging's input-norm pass: inverse RMS per staged token
// row and the consumer warps' partial sums of squares (128-byte granule).
__host__ __device__ constexpr size_t gemv_norm_bytes(int consumer_warps) {
  return ((size_t)kGemvNormTokens * (1 + consumer_warps) * 4 + 127) / 128 * 128;
}

// Tensor maps of one K-split matrix: codes (u64 elements), scales, mins (u16;
// INT4 only).
struct QWMaps {
  CUtensorMap codes, scale, mn;
};

struct TmaGemvArgs {
  // K-split jobs load [R rows] x [ks_len] boxes through 2-D tensor maps:
  QWMaps dmap;                 // dense mode (kernel parameter)
  const QWMaps* maps;          // grouped mode: per expert, device memory
  const QWMaps* maps_s;        // shared job, device memory
  int use_maps;                // 1: tensor maps; 0: 1-D bulk copies of whole rows
  int fmt, act;
  QW a0, a1;                   // dense mode: matrices (a1: up, when fused)
  const QW* tab0;              // grouped mode: per-expert tables (device)
  const QW* tab1;
  QW s0, s1;                   // shared expert matrices
  int N, K;                    // dense / routed rows and reduction width
  int Ns, Ks;                  // shared rows and width
  const uint16_t* x;           // dense / routed input rows
  int ld_x;                    // row stride of x (elements)
  const uint16_t* x_s;         // shared job input rows (row stride Ks)
  int M, topk;
  const int* perm;             // routed gate/up: input row of slot s = perm[s] / topk
  const int* offsets;          // null: dense mode
  const int* union_list;
  const int* n_union;
  int routed_jobs;
  int slots;                   // slot count of out_d (dense: M, routed: M*topk)
  uint16_t* out_act;           // fused gate/up: [slots][N] bf16
  uint16_t* out_act_s;         // [M][Ns]
  float* out_d;                // down: [splits][slots][N] fp32 partial sums
  float* out_d_s;              // [splits][M][N]
  int* zero_cnt;               // gate/up, dense mode: counters cleared for the down launch that follows
  int zero_n;
  int* tile_cnt;               // down, dense mode: arrivals of the K splits per CTA row range
  uint16_t* res;               // down, dense mode: residual [M][N], updated in place by the last K split
                               // of each row range (null: fp32 partials only, a tail kernel adds them)
  const uint16_t* norm_w;      // dense gate/up, unsplit K: normalize x on staging (RMSNorm weight [K]), or null
  float eps;
  int ks_len;                  // K elements per split (INT4, Q4_K: multiple of 256)
  int ctas_per_job;
  int stage_tokens;
  int stages;
  // Failure-detection tests only (0 in every product launch): the producer
  // issues no stage from index inject_stop - 1 on, as if it had died, and the
  // pipeline waits give up after wait_ns (0: the default of about a second).
  int inject_stop;
  unsigned long long wait_ns;
};

// Encodes the three maps of W[N][K] for boxes of [rows_per_stage][ks_len].
cudaError_t encode_qw_maps(QWMaps* m, int fmt, const QW& w, int N, int K, int ks_len);
// nm: 2 for the fused gate/up launch, 1 for a single matrix (the down
// projection), whose stages hold row pairs: 2 x 8 rows, the bytes of a
// two-matrix stage, so its geometry is that of nm = 2.
size_t tma_gemv_smem(int fmt, int nm, int klen, int stage_tokens, int mt, int stages);
size_t tma_gemv_stage_bytes(int fmt, int nm, int klen);
cudaError_t launch_tma_gemv(const TmaGemvArgs& a, int nm, int mt, int splits, int jobs, cudaStream_t s);
unsigned int tma_gemv_fault_flags(bool clear);

}  // namespace moeffn
