// Test exports: single steps of the path fed with caller-chosen inputs, so
// that the bit-exact parts (dequantization, top-k, permutation) can be
// compared with the oracle on identical inputs.
#include <string>

#include "../../include/moeffn.h"
#include "common.cuh"
#include "route.cuh"

using namespace moeffn;

namespace moeffn {
int api_fail(int code, const char* msg);
}

namespace {

__device__ int g_test_route_counter = 0;   // arrival counter of the test export's top-k CTAs

// One thread per 32-bit word of codes: 8 INT4 codes or 4 INT8 codes.
__global__ void k_dequant(const QW w, int fmt, int N, int K, float* out_f32, uint16_t* out_bf16) {
  const int per_word = fmt == FMT_INT4_G32 ? 8 : 4;
  const size_t words = (size_t)N * K / per_word;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < words; i += (size_t)gridDim.x * blockDim.x) {
    const uint32_t word = reinterpret_cast<const uint32_t*>(w.q)[i];
    const size_t e0 = i * per_word;
    const int n = (int)(e0 / K), k0 = (int)(e0 - (size_t)n * K);
    float v[8];
    if (fmt == FMT_INT4_G32) {
      const float s = __half2float(w.scale[(size_t)n * (K / 32) + k0 / 32]);
      const float m = __half2float(w.mn[(size_t)n * (K / 32) + k0 / 32]);
      int4_word_dequant(word, s, m, v);
    } else {
      float v4[4];
      int8_word_dequant(word, __half2float(w.scale[n]), v4);
      for (int j = 0; j < 4; ++j) v[j] = v4[j];
    }
    for (int j = 0; j < per_word; ++j) {
      if (out_f32) out_f32[e0 + j] = v[j];
      if (out_bf16) out_bf16[e0 + j] = float_to_bf16_bits(v[j]);
    }
  }
}

// Q4_K: one thread per code word (4 bytes of a run): weights 64c + 4v .. + 3
// of the low sub-block and the same + 32 of the high one, each
// fmaf(q, d * scale, -dmin * min) as in the GEMV and GEMM.
__global__ void k_dequant_q4k(const uint8_t* q, int N, int K, float* out_f32, uint16_t* out_bf16) {
  const size_t words = (size_t)N * (K / Q4K::kBlock) * 32;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < words; i += (size_t)gridDim.x * blockDim.x) {
    const size_t blk = i / 32;                   // block index over the whole matrix
    const int v = (int)(i % 32), c = v / 8;      // word v of the block's codes, in run c
    const uint8_t* b = q + blk * Q4K::kBytes;
    const uint4 hdr = *reinterpret_cast<const uint4*>(b);
    const uint32_t w = *reinterpret_cast<const uint32_t*>(b + 16 + 4 * v);
    float sl, ml, sh, mh;
    Q4K::scale_min(hdr, 2 * c, sl, ml);
    Q4K::scale_min(hdr, 2 * c + 1, sh, mh);
    const size_t e0 = blk * Q4K::kBlock + 64 * c + 4 * (v % 8);   // element index (row-major: blocks in order)
    for (int j = 0; j < 4; ++j) {
      const float lo = fmaf((float)((w >> (8 * j)) & 15u), sl, ml);
      const float hi = fmaf((float)((w >> (8 * j + 4)) & 15u), sh, mh);
      if (out_f32) { out_f32[e0 + j] = lo; out_f32[e0 + 32 + j] = hi; }
      if (out_bf16) { out_bf16[e0 + j] = float_to_bf16_bits(lo); out_bf16[e0 + 32 + j] = float_to_bf16_bits(hi); }
    }
  }
}

}  // namespace

extern "C" {

int moeffn_test_dequant(const moeffn_qweight* w, float* out_f32, uint16_t* out_bf16, moeffn_stream_t stream) {
  if (w != nullptr && w->format == MOEFFN_Q_Q4_K) {
    if (w->q == nullptr) return api_fail(MOEFFN_ERR_INVALID, "test_dequant: null");
    if (w->rows < 1 || w->cols < 256 || w->cols % 256 != 0) return api_fail(MOEFFN_ERR_INVALID, "test_dequant: shape");
    if ((reinterpret_cast<uintptr_t>(w->q) & 15u) != 0) return api_fail(MOEFFN_ERR_INVALID, "test_dequant: q misaligned");
    k_dequant_q4k<<<296, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(static_cast<const uint8_t*>(w->q), w->rows,
                                                                          w->cols, out_f32, out_bf16);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return api_fail(MOEFFN_ERR_CUDA, cudaGetErrorString(e));
    return MOEFFN_OK;
  }
  if (w == nullptr || w->q == nullptr || w->scale == nullptr) return api_fail(MOEFFN_ERR_INVALID, "test_dequant: null");
  if (w->format != MOEFFN_Q_INT8_ROW && w->format != MOEFFN_Q_INT4_AFFINE_G32)
    return api_fail(MOEFFN_ERR_UNSUPPORTED, "test_dequant: format");
  if (w->rows < 1 || w->cols < 1 || w->cols % (w->format == MOEFFN_Q_INT4_AFFINE_G32 ? 32 : 16) != 0)
    return api_fail(MOEFFN_ERR_INVALID, "test_dequant: shape");
  if (w->format == MOEFFN_Q_INT4_AFFINE_G32 && w->min == nullptr) return api_fail(MOEFFN_ERR_INVALID, "test_dequant: min");
  if ((reinterpret_cast<uintptr_t>(w->q) & 3u) != 0) return api_fail(MOEFFN_ERR_INVALID, "test_dequant: q misaligned");
  const QW q{static_cast<const uint8_t*>(w->q), static_cast<const __half*>(w->scale),
             static_cast<const __half*>(w->min)};
  k_dequant<<<296, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(q, w->format, w->rows, w->cols, out_f32, out_bf16);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return api_fail(MOEFFN_ERR_CUDA, cudaGetErrorString(e));
  return MOEFFN_OK;
}

int moeffn_test_topk_from_logits(const float* logits, int M, int E, int top_k, int32_t* topk_idx, float* topk_w,
                                 int32_t* perm, int32_t* expert_offsets, int32_t* union_out, int32_t* n_union_out,
                                 moeffn_stream_t stream) {
  if (logits == nullptr || topk_idx == nullptr || topk_w == nullptr) return api_fail(MOEFFN_ERR_INVALID, "test_topk: null");
  if (M < 1 || E < 1 || E > kMaxExperts || top_k < 1 || top_k > kMaxTopK || top_k > E)
    return api_fail(MOEFFN_ERR_INVALID, "test_topk: sizes");
  if (perm != nullptr && expert_offsets == nullptr) return api_fail(MOEFFN_ERR_INVALID, "test_topk: perm needs offsets");
  RouteArgs a{};
  a.logits = logits;
  a.M = M;
  a.E = E;
  a.k = top_k;
  a.idx = topk_idx;
  a.w = topk_w;
  a.perm = perm;
  a.offsets = expert_offsets;
  a.union_list = union_out;
  a.n_union = n_union_out;
  // The top-k CTAs count their arrivals in a counter that must start at zero.
  static int* counter[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return api_fail(MOEFFN_ERR_CUDA, "test_topk: device");
  if (counter[dev] == nullptr && cudaGetSymbolAddress(reinterpret_cast<void**>(&counter[dev]), g_test_route_counter) != cudaSuccess)
    return api_fail(MOEFFN_ERR_CUDA, "test_topk: counter address");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(counter[dev], 0, sizeof(int), st) != cudaSuccess) return api_fail(MOEFFN_ERR_CUDA, "test_topk: memset");
  a.counter = counter[dev];
  const cudaError_t e = launch_route(a, st);
  if (e != cudaSuccess) return api_fail(MOEFFN_ERR_CUDA, cudaGetErrorString(e));
  return MOEFFN_OK;
}

}  // extern "C"
