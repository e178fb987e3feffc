// Layer tails that consume the down projection's fp32 partial sums:
//
//  * residual : x = bf16(x + bf16(h))  -- the llama dense layer's raw residual
//               add (turbospark-runtime 0.3.0, src/families/llama/dense.rs,
//               encode_llama_layer_dense: down GEMV into h2, then residual add);
//  * rmsnorm  : h1 = bf16(h); h1 = bf16(h1 / sqrt(mean(h1^2) + eps) * w), in
//               place -- the Gemma shared-expert branch's trailing
//               post_feedforward_layernorm_1 (turbospark-runtime 0.1.0,
//               src/families/gemma4/shared_expert.rs);
//  * moe      : acc = seed; acc += w_r * d_r for r = 0..k-1 in rank order;
//               x = bf16(x + bf16(acc)) -- the seeded phase-2 reduction and the
//               single raw residual add of turbospark-runtime 0.3.0,
//               src/families/qwen/moe_batch.rs (module doc: the accumulator is
//               seeded with the gated shared expert; no norm in the tail).
//               seed = bf16(bf16(s) * sigmoid(gate_logit)) with s the shared
//               expert's down output, or 0 without a shared expert.
//  * moe, Gemma form: the routed sum starts from 0; the shared branch joins
//               after its post-FFN norm: h1 = bf16(RMSNorm(bf16(s)) * w),
//               x = bf16(x + bf16(y + h1)) (turbospark-runtime 0.3.0,
//               src/families/qwen/moe_batch.rs, module doc on Gemma; the
//               branch norm of turbospark-runtime 0.1.0,
//               src/families/gemma4/shared_expert.rs).
#include "launch.cuh"
#include "tail.cuh"

namespace moeffn {

namespace {

__device__ __forceinline__ float sum_splits(const float* d, int splits, size_t split_stride, size_t off) {
  float h = 0.f;
  for (int s = 0; s < splits; ++s) h += d[s * split_stride + off];   // fixed split order
  return h;
}

__global__ void k_tail_elementwise(const TailArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t total = (size_t)a.M * a.N;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / a.N), n = (int)(i - (size_t)t * a.N);
    float y;
    if (a.mode == TAIL_RESIDUAL) {
      y = round_bf16(sum_splits(a.d, a.splits, (size_t)a.slots * a.N, (size_t)t * a.N + n));
    } else {
      float acc = 0.f;
      if (a.d_s != nullptr) {
        const float s = round_bf16(sum_splits(a.d_s, a.splits_s, (size_t)a.M * a.N, (size_t)t * a.N + n));
        acc = round_bf16(s * sigmoid_f(a.gate_logit[t]));
      }
      for (int r = 0; r < a.k; ++r) {
        const int slot = a.inv[t * a.k + r];
        const float dr = sum_splits(a.d, a.splits, (size_t)a.slots * a.N, (size_t)slot * a.N + n);
        acc = __fadd_rn(acc, __fmul_rn(a.w[t * a.k + r], dr));
      }
      y = round_bf16(acc);
    }
    const float x = bf16_bits_to_float(a.res[i]);
    a.res[i] = float_to_bf16_bits(x + y);
  }
}

__global__ void __launch_bounds__(512) k_tail_rmsnorm(const TailArgs a) {
  extern __shared__ float red[];
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  float ss = 0.f;
  for (int n = threadIdx.x; n < a.N; n += blockDim.x) {
    const float h = round_bf16(sum_splits(a.d, a.splits, (size_t)a.slots * a.N, (size_t)t * a.N + n));
    ss = fmaf(h, h, ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float inv_rms = 1.0f / sqrtf(red[0] / (float)a.N + a.eps);
  for (int n = threadIdx.x; n < a.N; n += blockDim.x) {
    const float h = round_bf16(sum_splits(a.d, a.splits, (size_t)a.slots * a.N, (size_t)t * a.N + n));
    const float w = bf16_bits_to_float(a.norm_w[n]);
    a.h1[(size_t)t * a.N + n] = float_to_bf16_bits(h * inv_rms * w);
  }
}

// Gemma-form MoE tail, one CTA per token row: the shared branch's RMSNorm
// needs the whole row of its output first.
__global__ void __launch_bounds__(512) k_tail_moe_gemma(const TailArgs a) {
  __shared__ float red[16];
  pdl_launch_dependents();
  pdl_wait();
  const int t = blockIdx.x;
  const size_t sstride = (size_t)a.M * a.N;
  float ss = 0.f;
  for (int n = threadIdx.x; n < a.N; n += blockDim.x) {
    const float h = round_bf16(sum_splits(a.d_s, a.splits_s, sstride, (size_t)t * a.N + n));
    ss = fmaf(h, h, ss);
  }
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  const float inv_rms = 1.0f / sqrtf(red[0] / (float)a.N + a.eps);
  for (int n = threadIdx.x; n < a.N; n += blockDim.x) {
    const size_t o = (size_t)t * a.N + n;
    const float h = round_bf16(sum_splits(a.d_s, a.splits_s, sstride, o));
    const float h1 = round_bf16(h * inv_rms * bf16_bits_to_float(a.norm_w[n]));
    float acc = 0.f;   // the routed sum starts from nothing
    for (int r = 0; r < a.k; ++r) {
      const int slot = a.inv[t * a.k + r];
      const float dr = sum_splits(a.d, a.splits, (size_t)a.slots * a.N, (size_t)slot * a.N + n);
      acc = __fadd_rn(acc, __fmul_rn(a.w[t * a.k + r], dr));
    }
    const float y = round_bf16(acc);
    a.res[o] = float_to_bf16_bits(bf16_bits_to_float(a.res[o]) + round_bf16(y + h1));
  }
}

}  // namespace

cudaError_t launch_tail(const TailArgs& a, cudaStream_t s) {
  if (a.mode == TAIL_MOE_GEMMA) {
    return launch_pdl(k_tail_moe_gemma, dim3(a.M), dim3(512), 0, s, a);
  }
  if (a.mode == TAIL_RMSNORM) {
    return launch_pdl(k_tail_rmsnorm, dim3(a.M), dim3(512), 16 * sizeof(float), s, a);
  } else {
    const size_t total = (size_t)a.M * a.N;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 148 * 8) blocks = 148 * 8;
    return launch_pdl(k_tail_elementwise, dim3(blocks), dim3(256), 0, s, a);
  }
  return cudaGetLastError();
}

}  // namespace moeffn
