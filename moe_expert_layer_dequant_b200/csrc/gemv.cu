// Weight-streaming GEMV kernels for few token rows (decode): the fused
// gate/up projection with the gated activation in its epilogue, and the down
// projection split along K into fp32 partial sums.
//
// Each warp owns whole weight rows; each lane streams 16-byte chunks of a row
// (one INT4 group of 32 codes, or 16 INT8 codes) with 128-bit loads, turns the
// codes into floats in registers and multiplies them with activations staged
// once per CTA in shared memory. Row sums are finished with warp shuffles.
//
// The same kernels serve three kinds of work ("jobs"), selected by blockIdx.y:
//  * dense       : one matrix, tokens 0..M-1 (the llama dense FFN and the
//                  Gemma shared-expert branch);
//  * routed job u: expert union[u] of the MoE layer, over the (token, rank)
//                  pairs routed to it, read and written in expert-grouped
//                  slot order;
//  * shared job  : the MoE layer's shared expert, over all M tokens.
#include "gemv.cuh"
#include "launch.cuh"

namespace moeffn {

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kUnroll = 4;  // 16-byte chunks in flight per lane per matrix

template <int FMT>
struct Fmt;
template <>
struct Fmt<FMT_INT4_G32> {
  static constexpr int kChunk = 32;  // elements per 16-byte chunk
  static constexpr bool kGroups = true;
  static __device__ __forceinline__ float pos_scale(int k) { return int4_pos_scale(k); }
};
template <>
struct Fmt<FMT_INT8_ROW> {
  static constexpr int kChunk = 16;
  static constexpr bool kGroups = false;
  static __device__ __forceinline__ float pos_scale(int k) { return int8_pos_scale(k); }
};

// Padded chunk stride in shared memory (floats): a 16-byte pad after every
// chunk keeps the lanes' 128-bit reads of different chunks on distinct banks.
template <int FMT>
__host__ __device__ constexpr int chunk_stride() {
  return (FMT == FMT_INT4_G32 ? 32 : 16) + 4;
}

// Stage token rows [k0, k0+klen) of bf16 activations as position-scaled fp32,
// plus (INT4) the plain per-group sums. Row r of the stage reads src row
// row_of(r).
template <int FMT, class RowOf>
__device__ void stage_rows(float* xs, float* xsum, const uint16_t* __restrict__ src, int ld, int k0,
                           int klen, int nrows, RowOf row_of) {
  constexpr int CE = Fmt<FMT>::kChunk;
  constexpr int CS = chunk_stride<FMT>();
  const int nch = klen / CE;
  const int tok_stride = nch * CS;
  const int per_row = klen / 8;
  for (int i = threadIdx.x; i < nrows * per_row; i += blockDim.x) {
    const int r = i / per_row;
    const int kk = (i - r * per_row) * 8;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (size_t)row_of(r) * ld + k0 + kk);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const int c = kk / CE, o = kk - c * CE;
    float* dst = xs + r * tok_stride + c * CS + o;
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[2 * j] = __uint_as_float(w[j] << 16) * Fmt<FMT>::pos_scale(kk + 2 * j);
      f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u) * Fmt<FMT>::pos_scale(kk + 2 * j + 1);
    }
    *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
  }
  if (Fmt<FMT>::kGroups) {
    const int ng = klen / 32;
    for (int i = threadIdx.x; i < nrows * ng; i += blockDim.x) {
      const int r = i / ng, g = i - r * ng;
      const uint16_t* p = src + (size_t)row_of(r) * ld + k0 + g * 32;
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = *reinterpret_cast<const uint4*>(p + 8 * q);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) s += __uint_as_float(w[j] << 16) + __uint_as_float(w[j] & 0xFFFF0000u);
      }
      xsum[r * ng + g] = s;
    }
  }
}

// Dot products of NM weight rows (same row index n of NM matrices) with MT
// staged token rows over chunks [c_lo, c_hi) of the full row (chunk indices
// relative to the staged slice start at c_base). Per-lane partial results.
template <int FMT, int MT, int NM>
__device__ __forceinline__ void row_dots(const QW (&m)[NM], int n, int K, int c_base, int c_hi,
                                         const float* xs, int tok_stride, const float* xsum, int ng_slice,
                                         int tvalid, float (&acc)[NM][MT]) {
  constexpr int CS = chunk_stride<FMT>();
  const int lane = threadIdx.x & 31;
  const int row_bytes = (FMT == FMT_INT4_G32) ? K / 2 : K;
  const int groups = K / 32;
#pragma unroll
  for (int i = 0; i < NM; ++i)
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[i][t] = 0.f;

  for (int c0 = c_base + lane; c0 < c_hi; c0 += 32 * kUnroll) {
    uint4 wv[NM][kUnroll];
    float sc[NM][kUnroll], mn[NM][kUnroll];
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const int c = c0 + 32 * j;
      if (c < c_hi) {
#pragma unroll
        for (int i = 0; i < NM; ++i) {
          wv[i][j] = ld_stream_u4(m[i].q + (size_t)n * row_bytes + (size_t)c * 16);
          if (FMT == FMT_INT4_G32) {
            sc[i][j] = __half2float(m[i].scale[(size_t)n * groups + c]);
            mn[i][j] = __half2float(m[i].mn[(size_t)n * groups + c]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kUnroll; ++j) {
      const int c = c0 + 32 * j;
      if (c >= c_hi) break;
      const int cl = c - c_base;
#pragma unroll
      for (int i = 0; i < NM; ++i) {
        const uint32_t w[4] = {wv[i][j].x, wv[i][j].y, wv[i][j].z, wv[i][j].w};
        float2 p[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) p[t] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (FMT == FMT_INT4_G32) {
            float2 cf[4];
            int4_word_codes(w[q], cf);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (t < tvalid) {
                const float* xp = xs + t * tok_stride + cl * CS + 8 * q;
                const float4 xa = *reinterpret_cast<const float4*>(xp);
                const float4 xb = *reinterpret_cast<const float4*>(xp + 4);
                p[t] = __ffma2_rn(cf[0], make_float2(xa.x, xa.y), p[t]);
                p[t] = __ffma2_rn(cf[1], make_float2(xa.z, xa.w), p[t]);
                p[t] = __ffma2_rn(cf[2], make_float2(xb.x, xb.y), p[t]);
                p[t] = __ffma2_rn(cf[3], make_float2(xb.z, xb.w), p[t]);
              }
            }
          } else {
            float2 cf[2];
            int8_word_codes(w[q], cf);
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              if (t < tvalid) {
                const float4 xa = *reinterpret_cast<const float4*>(xs + t * tok_stride + cl * CS + 4 * q);
                p[t] = __ffma2_rn(cf[0], make_float2(xa.x, xa.y), p[t]);
                p[t] = __ffma2_rn(cf[1], make_float2(xa.z, xa.w), p[t]);
              }
            }
          }
        }
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (t < tvalid) {
            const float P = p[t].x + p[t].y;
            if (FMT == FMT_INT4_G32) {
              // sum_i (q_i s + m) x_i = s * sum_i q_i x_i + m * sum_i x_i
              acc[i][t] = fmaf(sc[i][j], P, fmaf(mn[i][j], xsum[t * ng_slice + cl], acc[i][t]));
            } else {
              acc[i][t] += P;
            }
          }
        }
      }
    }
  }
}

struct Job {
  QW a, b;
  int N;        // rows of the job's matrices
  int K;        // reduction width of the job's matrices
  int ntok;     // token rows of the job
  int slot0;    // first output slot (grouped) or 0
  bool gather;  // input row of token j is perm[slot0 + j] / topk
  bool valid;
};

__device__ __forceinline__ Job gateup_job(const GateUpArgs& a) {
  Job j{};
  j.valid = true;
  j.K = a.K;
  const int job = blockIdx.y;
  if (a.perm == nullptr) {
    j.a = a.g; j.b = a.u; j.N = a.N; j.ntok = a.M;
  } else if (job < a.routed_jobs) {
    if (job >= *a.n_union) { j.valid = false; return j; }
    const int e = a.union_list[job];
    j.a = a.g_tab[e]; j.b = a.u_tab[e]; j.N = a.N;
    j.slot0 = a.offsets[e];
    j.ntok = a.offsets[e + 1] - j.slot0;
    j.gather = true;
  } else {
    j.a = a.sg; j.b = a.su; j.N = a.Ns; j.ntok = a.M;
  }
  return j;
}

template <int FMT, int MT>
__global__ void __launch_bounds__(kThreads, 2) k_gateup(const GateUpArgs a) {
  extern __shared__ __align__(16) float smem[];
  pdl_launch_dependents();
  pdl_wait();
  const Job job = gateup_job(a);
  if (!job.valid) return;
  const int row0 = blockIdx.x * a.rows_per_cta;
  if (row0 >= job.N || job.ntok == 0) return;
  const int row1 = min(job.N, row0 + a.rows_per_cta);
  uint16_t* out = (a.perm != nullptr && blockIdx.y >= a.routed_jobs) ? a.out_s : a.out;

  constexpr int CE = Fmt<FMT>::kChunk;
  const int nch = job.K / CE;
  const int tok_stride = nch * chunk_stride<FMT>();
  const int ng = job.K / 32;
  float* xs = smem;
  float* xsum = smem + a.stage_tokens * tok_stride;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const QW mats[2] = {job.a, job.b};

  for (int t0 = 0; t0 < job.ntok; t0 += a.stage_tokens) {
    const int tn = min(a.stage_tokens, job.ntok - t0);
    __syncthreads();
    stage_rows<FMT>(xs, xsum, a.x, a.K, 0, job.K, tn, [&](int r) {
      return job.gather ? a.perm[job.slot0 + t0 + r] / a.topk : t0 + r;
    });
    __syncthreads();
    for (int n = row0 + warp; n < row1; n += kWarps) {
      for (int tc = 0; tc < tn; tc += MT) {
        float acc[2][MT];
        row_dots<FMT, MT, 2>(mats, n, job.K, 0, nch, xs + tc * tok_stride, tok_stride, xsum + tc * ng, ng,
                             tn - tc, acc);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          float g = warp_sum(acc[0][t]);
          float u = warp_sum(acc[1][t]);
          if (lane == 0 && tc + t < tn) {
            if (FMT == FMT_INT8_ROW) {
              g *= __half2float(job.a.scale[n]);
              u *= __half2float(job.b.scale[n]);
            }
            out[(size_t)(job.slot0 + t0 + tc + t) * job.N + n] = float_to_bf16_bits(gated_act(g, u, a.act));
          }
        }
      }
    }
  }
}

__device__ __forceinline__ Job down_job(const DownArgs& a) {
  Job j{};
  j.valid = true;
  const int job = blockIdx.z;
  if (a.offsets == nullptr) {
    j.a = a.w; j.N = a.N; j.K = a.K; j.ntok = a.M;
  } else if (job < a.routed_jobs) {
    if (job >= *a.n_union) { j.valid = false; return j; }
    const int e = a.union_list[job];
    j.a = a.tab[e]; j.N = a.N; j.K = a.K;
    j.slot0 = a.offsets[e];
    j.ntok = a.offsets[e + 1] - j.slot0;
  } else {
    j.a = a.ws; j.N = a.N; j.K = a.Ks; j.ntok = a.M;
  }
  return j;
}

template <int FMT, int MT>
__global__ void __launch_bounds__(kThreads, 2) k_down(const DownArgs a) {
  extern __shared__ __align__(16) float smem[];
  pdl_launch_dependents();
  pdl_wait();
  const Job job = down_job(a);
  if (!job.valid || job.ntok == 0) return;
  const bool shared_job = (a.offsets != nullptr && blockIdx.z >= a.routed_jobs);
  const int row0 = blockIdx.x * a.rows_per_cta;
  const int row1 = min(job.N, row0 + a.rows_per_cta);
  const int k0 = blockIdx.y * a.ks_len;
  if (row0 >= job.N || k0 >= job.K) return;
  const int klen = min(a.ks_len, job.K - k0);
  const uint16_t* in = shared_job ? a.in_s : a.in;
  float* d = shared_job ? a.d_s : a.d;
  const int nslots = shared_job ? a.M : a.slots;

  constexpr int CE = Fmt<FMT>::kChunk;
  const int nch = klen / CE;
  const int tok_stride = nch * chunk_stride<FMT>();
  const int ng = klen / 32;
  float* xs = smem;
  float* xsum = smem + a.stage_tokens * tok_stride;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const QW mats[1] = {job.a};
  const int c_base = k0 / CE;

  for (int t0 = 0; t0 < job.ntok; t0 += a.stage_tokens) {
    const int tn = min(a.stage_tokens, job.ntok - t0);
    __syncthreads();
    stage_rows<FMT>(xs, xsum, in, job.K, k0, klen, tn, [&](int r) { return job.slot0 + t0 + r; });
    __syncthreads();
    for (int n = row0 + warp; n < row1; n += kWarps) {
      const float rs = (FMT == FMT_INT8_ROW) ? __half2float(job.a.scale[n]) : 1.0f;
      for (int tc = 0; tc < tn; tc += MT) {
        float acc[1][MT];
        row_dots<FMT, MT, 1>(mats, n, job.K, c_base, c_base + nch, xs + tc * tok_stride, tok_stride,
                             xsum + tc * ng, ng, tn - tc, acc);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const float h = warp_sum(acc[0][t]);
          if (lane == 0 && tc + t < tn)
            d[((size_t)blockIdx.y * nslots + job.slot0 + t0 + tc + t) * job.N + n] = h * rs;
        }
      }
    }
  }
}

template <int FMT>
int stage_floats_per_token(int klen) {
  return (klen / Fmt<FMT>::kChunk) * chunk_stride<FMT>() + (FMT == FMT_INT4_G32 ? klen / 32 : 0);
}

template <class Args, class KernelT>
cudaError_t launch(KernelT kern, dim3 grid, size_t smem, cudaStream_t s, const Args& a) {
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(kern, grid, dim3(kThreads), smem, s, a);
}

}  // namespace

size_t gemv_stage_bytes(int fmt, int klen, int tokens) {
  // (Q4_K rows stage like INT4 rows: 32-element chunks with sums)
  const int per = fmt == FMT_INT8_ROW ? stage_floats_per_token<FMT_INT8_ROW>(klen)
                                      : stage_floats_per_token<FMT_INT4_G32>(klen);
  return (size_t)per * tokens * sizeof(float);
}

cudaError_t launch_gateup(const GateUpArgs& a, int grid_x, int jobs, int mt, cudaStream_t s) {
  const size_t smem = gemv_stage_bytes(a.fmt, a.K, a.stage_tokens);
  const dim3 grid(grid_x, jobs);
  if (a.fmt == FMT_INT4_G32)
    return mt == 1 ? launch(k_gateup<FMT_INT4_G32, 1>, grid, smem, s, a)
                   : launch(k_gateup<FMT_INT4_G32, 2>, grid, smem, s, a);
  return mt == 1 ? launch(k_gateup<FMT_INT8_ROW, 1>, grid, smem, s, a)
                 : launch(k_gateup<FMT_INT8_ROW, 2>, grid, smem, s, a);
}

cudaError_t launch_down(const DownArgs& a, int grid_x, int splits, int jobs, int mt, cudaStream_t s) {
  const size_t smem = gemv_stage_bytes(a.fmt, a.ks_len, a.stage_tokens);
  const dim3 grid(grid_x, splits, jobs);
  if (a.fmt == FMT_INT4_G32)
    return mt == 1 ? launch(k_down<FMT_INT4_G32, 1>, grid, smem, s, a)
                   : launch(k_down<FMT_INT4_G32, 2>, grid, smem, s, a);
  return mt == 1 ? launch(k_down<FMT_INT8_ROW, 1>, grid, smem, s, a)
                 : launch(k_down<FMT_INT8_ROW, 2>, grid, smem, s, a);
}

}  // namespace moeffn
