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

// Four consecutive features per thread (16-byte partial loads); N % 4 == 0.
// KMAX: a bound on top-k (2, 4, 8 or 16), so that the per-rank registers stay few.
template <int KMAX>
__global__ void k_tail_elementwise(const TailArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t total4 = (size_t)a.M * a.N / 4;
  const size_t rstride = (size_t)a.slots * a.N, sstride = (size_t)a.M * a.N;
  for (size_t i4 = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i4 < total4; i4 += (size_t)gridDim.x * blockDim.x) {
    const size_t i = 4 * i4;
    const int t = (int)(i / a.N), n = (int)(i - (size_t)t * a.N);
    float y[4];
    if (a.mode == TAIL_RESIDUAL) {
      float4 h = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int sp = 0; sp < a.splits; ++sp) {   // fixed split order
        const float4 v = *reinterpret_cast<const float4*>(a.d + sp * rstride + (size_t)t * a.N + n);
        h.x += v.x; h.y += v.y; h.z += v.z; h.w += v.w;
      }
      y[0] = round_bf16(h.x); y[1] = round_bf16(h.y); y[2] = round_bf16(h.z); y[3] = round_bf16(h.w);
    } else {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
      if (a.d_s != nullptr) {
        float4 sh = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < a.splits_s; ++sp) {
          const float4 v = *reinterpret_cast<const float4*>(a.d_s + sp * sstride + (size_t)t * a.N + n);
          sh.x += v.x; sh.y += v.y; sh.z += v.z; sh.w += v.w;
        }
        const float g = sigmoid_f(a.gate_logit[t]);
        acc[0] = round_bf16(round_bf16(sh.x) * g); acc[1] = round_bf16(round_bf16(sh.y) * g);
        acc[2] = round_bf16(round_bf16(sh.z) * g); acc[3] = round_bf16(round_bf16(sh.w) * g);
      }
      // All ranks' slots and weights first, then every rank's partials split
      // by split (the loads of one split are independent), then the sum:
      // seed first, then the ranks in order; each rank's splits in order.
      int slot[KMAX];
      float wr[KMAX];
      float4 d[KMAX];
#pragma unroll
      for (int r = 0; r < KMAX; ++r) {
        d[r] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (r < a.k) { slot[r] = a.inv[t * a.k + r]; wr[r] = a.w[t * a.k + r]; }
      }
      for (int sp = 0; sp < a.splits; ++sp) {
#pragma unroll
        for (int r = 0; r < KMAX; ++r) {
          if (r < a.k) {
            const float4 v = *reinterpret_cast<const float4*>(a.d + sp * rstride + (size_t)slot[r] * a.N + n);
            d[r].x += v.x; d[r].y += v.y; d[r].z += v.z; d[r].w += v.w;
          }
        }
      }
#pragma unroll
      for (int r = 0; r < KMAX; ++r) {
        if (r < a.k) {
          acc[0] = __fadd_rn(acc[0], __fmul_rn(wr[r], d[r].x)); acc[1] = __fadd_rn(acc[1], __fmul_rn(wr[r], d[r].y));
          acc[2] = __fadd_rn(acc[2], __fmul_rn(wr[r], d[r].z)); acc[3] = __fadd_rn(acc[3], __fmul_rn(wr[r], d[r].w));
        }
      }
      for (int j = 0; j < 4; ++j) y[j] = round_bf16(acc[j]);
    }
    const uint2 rv = *reinterpret_cast<const uint2*>(a.res + i);
    const uint32_t r01 = rv.x, r23 = rv.y;
    const float x0 = __uint_as_float(r01 << 16), x1 = __uint_as_float(r01 & 0xFFFF0000u);
    const float x2 = __uint_as_float(r23 << 16), x3 = __uint_as_float(r23 & 0xFFFF0000u);
    uint2 ov;
    ov.x = (uint32_t)float_to_bf16_bits(x0 + y[0]) | ((uint32_t)float_to_bf16_bits(x1 + y[1]) << 16);
    ov.y = (uint32_t)float_to_bf16_bits(x2 + y[2]) | ((uint32_t)float_to_bf16_bits(x3 + y[3]) << 16);
    *reinterpret_cast<uint2*>(a.res + i) = ov;
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
    if (a.N % 4 != 0) return cudaErrorInvalidValue;
    const size_t total4 = (size_t)a.M * a.N / 4;
    // Small row counts: 128-thread blocks over more SMs; else 256.
    const int threads = total4 < (size_t)148 * 256 ? 128 : 256;
    int blocks = (int)((total4 + threads - 1) / threads);
    if (blocks > 148 * 8) blocks = 148 * 8;
    const int k = a.mode == TAIL_RESIDUAL ? 1 : a.k;
    if (k <= 2) return launch_pdl(k_tail_elementwise<2>, dim3(blocks), dim3(threads), 0, s, a);
    if (k <= 4) return launch_pdl(k_tail_elementwise<4>, dim3(blocks), dim3(threads), 0, s, a);
    if (k <= 8) return launch_pdl(k_tail_elementwise<8>, dim3(blocks), dim3(threads), 0, s, a);
    if (k <= 16) return launch_pdl(k_tail_elementwise<16>, dim3(blocks), dim3(threads), 0, s, a);
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace moeffn
