// The FFN's input norm m = rms_norm(x, w) (the llama layer's
// post_attention_layernorm, applied by the layer instead of its caller):
// m[k] = bf16(x[k] * inv_rms * w[k]), inv_rms = 1 / sqrt(mean(x^2) + eps),
// computed in fp32 on the bf16 residual row x (the same norm as the Gemma
// branch's trailing RMSNorm). Shared by the kernels that fold it in.
#pragma once
#include "common.cuh"

namespace moeffn {

// One element of m from the bf16 bits of x and w and the row's inv_rms.
__device__ __forceinline__ uint16_t prenorm_elem(uint16_t xb, uint16_t wb, float inv_rms) {
  return float_to_bf16_bits(bf16_bits_to_float(xb) * inv_rms * bf16_bits_to_float(wb));
}

// This thread's part of the sum of squares of row x[0..H) (16-byte loads;
// H a multiple of 8), threads `tid` of `nthreads`.
__device__ __forceinline__ float row_sumsq_part(const uint16_t* x, int H, int tid, int nthreads) {
  float ss = 0.f;
  for (int k = tid * 8; k < H; k += nthreads * 8) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(x + k));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __uint_as_float(w[j] << 16), b = __uint_as_float(w[j] & 0xFFFF0000u);
      ss = fmaf(a, a, ss);
      ss = fmaf(b, b, ss);
    }
  }
  return ss;
}

__device__ __forceinline__ float inv_rms_of(float sumsq, int H, float eps) {
  return 1.0f / sqrtf(sumsq / (float)H + eps);
}

}  // namespace moeffn
