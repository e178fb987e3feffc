// Weight-streaming GEMV for few token rows, fed by the TMA bulk-copy engine.
//
// One producer warp streams stages of R consecutive weight rows (codes, and
// for INT4 the group scales and mins) from HBM into a ring of shared-memory
// stages with cp.async.bulk, each stage completing an mbarrier by byte count.
// R consumer warps each take one row of a stage (one row of every matrix of
// the job: gate and up together for the fused projection), dequantize the
// codes in registers and multiply them with the activations staged once per
// CTA in shared memory; row sums are finished with warp shuffles. Consumers
// release a stage through a second mbarrier, and the producer refills it.
//
// Compared to one 128-bit load per lane per chunk (gemv.cu), the copy engine
// keeps several stages of every SM's rows in flight without holding them in
// registers, and the code-to-float conversion is one LOP3 per code.
//
// Jobs (blockIdx.z), K slices (blockIdx.y) and CTAs of a job (blockIdx.x):
//  dense job   : one matrix set, token rows 0..M-1;
//  routed job u: the u-th expert of the MoE union, over its pairs (slot order);
//  shared job  : the MoE layer's shared expert over all M tokens.
// A CTA takes a contiguous range of the job's rows (a multiple of R rows).
#include "gemv_tma.cuh"
#include "sync.cuh"

namespace moeffn {

namespace {

template <int FMT>
struct Codes;

template <>
struct Codes<FMT_INT4_G32> {
  static constexpr int kChunk = 32;      // codes per 16-byte chunk (one group)
  static constexpr int kStride = 36;     // padded fp32 stride of a staged chunk
  static constexpr int kFloat2 = 4;      // float2 per 32-bit word
  static __device__ __forceinline__ float pos_scale(int k) { return int4_pos_scale(k); }
  // Positioned codes q_i * 16^(i%4) of one word: one LOP3 per code.
  static __device__ __forceinline__ void word(uint32_t w, float2 (&c)[4]) {
    const uint32_t hi = w >> 16;
    const uint32_t m0 = 0x000Fu, m1 = 0x00F0u, m2 = 0x0F00u, m3 = 0xF000u, mg = kMagic;
    float2 a, b, d, e;
    a.x = __uint_as_float(and_or(w, m0, mg));
    a.y = __uint_as_float(and_or(w, m1, mg));
    b.x = __uint_as_float(and_or(w, m2, mg));
    b.y = __uint_as_float(and_or(w, m3, mg));
    d.x = __uint_as_float(and_or(hi, m0, mg));
    d.y = __uint_as_float(and_or(hi, m1, mg));
    e.x = __uint_as_float(and_or(hi, m2, mg));
    e.y = __uint_as_float(and_or(hi, m3, mg));
    const float2 sub = make_float2(-kMagicF, -kMagicF);
    c[0] = __fadd2_rn(a, sub);
    c[1] = __fadd2_rn(b, sub);
    c[2] = __fadd2_rn(d, sub);
    c[3] = __fadd2_rn(e, sub);
  }
};

template <>
struct Codes<FMT_INT8_ROW> {
  static constexpr int kChunk = 16;
  static constexpr int kStride = 20;
  static constexpr int kFloat2 = 2;
  static __device__ __forceinline__ float pos_scale(int k) { return int8_pos_scale(k); }
  static __device__ __forceinline__ void word(uint32_t w, float2 (&c)[4]) {
    const uint32_t hi = w >> 16;
    const uint32_t m0 = 0x00FFu, m1 = 0xFF00u, x0 = 0x0080u | kMagic, x1 = 0x8000u | kMagic;
    float2 a, b;
    a.x = __uint_as_float(and_xor(w, m0, x0));
    a.y = __uint_as_float(and_xor(w, m1, x1));
    b.x = __uint_as_float(and_xor(hi, m0, x0));
    b.y = __uint_as_float(and_xor(hi, m1, x1));
    const float2 sub = make_float2(-(kMagicF + 128.0f), -(kMagicF + 32768.0f));
    c[0] = __fadd2_rn(a, sub);
    c[1] = __fadd2_rn(b, sub);
  }
};

struct Job {
  QW m[2];
  int N, K, ntok, slot0;
  bool gather, shared, valid;
};

__device__ __forceinline__ Job decode_job(const TmaGemvArgs& a) {
  Job j{};
  j.valid = true;
  const int z = blockIdx.z;
  if (a.offsets == nullptr) {
    j.m[0] = a.a0; j.m[1] = a.a1; j.N = a.N; j.K = a.K; j.ntok = a.M;
  } else if (z < a.routed_jobs) {
    if (z >= *a.n_union) { j.valid = false; return j; }
    const int e = a.union_list[z];
    j.m[0] = a.tab0[e];
    if (a.tab1 != nullptr) j.m[1] = a.tab1[e];
    j.N = a.N; j.K = a.K;
    j.slot0 = a.offsets[e];
    j.ntok = a.offsets[e + 1] - j.slot0;
    j.gather = a.perm != nullptr;
  } else {
    j.m[0] = a.s0; j.m[1] = a.s1; j.N = a.Ns; j.K = a.Ks; j.ntok = a.M; j.shared = true;
  }
  return j;
}

__device__ __forceinline__ void consumer_sync(int nthreads) {
  asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

template <int FMT, int MT, int NM, int NC>
__global__ void __launch_bounds__(32 * (NC + 1), 1) k_gemv_tma(const TmaGemvArgs a) {
  using C = Codes<FMT>;
  constexpr bool kInt4 = (FMT == FMT_INT4_G32);
  constexpr int R = NC;  // rows per stage: one per consumer warp
  extern __shared__ __align__(128) uint8_t smem[];

  const Job job = decode_job(a);
  if (!job.valid || job.ntok == 0) return;
  const int k0 = blockIdx.y * a.ks_len;
  if (k0 >= job.K) return;
  const int klen = min(a.ks_len, job.K - k0);
  const int rpc = ((job.N + a.ctas_per_job - 1) / a.ctas_per_job + R - 1) / R * R;
  const int r0 = blockIdx.x * rpc;
  const int r1 = min(job.N, r0 + rpc);
  if (r0 >= r1) return;

  // ---- shared memory carve ------------------------------------------------
  const int S = a.stages;
  const int cb = kInt4 ? klen / 2 : klen;        // code bytes per row
  const int gs = kInt4 ? klen / 32 : 0;          // groups per row
  const int nch = klen / C::kChunk;
  const int tok_stride = nch * C::kStride;
  const int tok_rows = (a.stage_tokens + MT - 1) / MT * MT;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + S;
  float* xs = reinterpret_cast<float*>(smem + 128);
  float* xsum = xs + tok_rows * tok_stride;
  const size_t x_bytes = ((size_t)tok_rows * (tok_stride + gs) * 4 + 127) / 128 * 128;
  uint8_t* stage0 = smem + 128 + x_bytes;
  const size_t stage_bytes = (size_t)NM * R * (cb + 4 * gs);
  // within a stage: codes [NM][R][cb], scales [NM][R][gs], mins [NM][R][gs]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NC);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int row_stages = (r1 - r0 + R - 1) / R;
  const int tok_blocks = (job.ntok + a.stage_tokens - 1) / a.stage_tokens;
  const int total = row_stages * tok_blocks;
  const int row_bytes = kInt4 ? job.K / 2 : job.K;
  const int row_groups = job.K / 32;

  if (warp == NC) {
    // ---------------- producer ----------------
    if (lane == 0) {
      for (int s = 0; s < total; ++s) {
        const int slot = s % S, use = s / S;
        if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1)) break;
        const int n0 = r0 + (s % row_stages) * R;
        const int nr = min(R, r1 - n0);
        uint8_t* st = stage0 + (size_t)slot * stage_bytes;
        mbar_arrive_expect_tx(&full[slot], (uint32_t)(NM * nr * (cb + 4 * gs)));
#pragma unroll
        for (int i = 0; i < NM; ++i) {
          const uint8_t* q = job.m[i].q + (size_t)n0 * row_bytes + (kInt4 ? k0 / 2 : k0);
          uint8_t* dq = st + (size_t)i * R * cb;
          if (klen == job.K) {
            bulk_g2s(dq, q, (uint32_t)(nr * cb), &full[slot]);
          } else {
            for (int r = 0; r < nr; ++r) bulk_g2s(dq + r * cb, q + (size_t)r * row_bytes, cb, &full[slot]);
          }
          if (kInt4) {
            const uint8_t* sc = reinterpret_cast<const uint8_t*>(job.m[i].scale) + ((size_t)n0 * row_groups + k0 / 32) * 2;
            const uint8_t* mn = reinterpret_cast<const uint8_t*>(job.m[i].mn) + ((size_t)n0 * row_groups + k0 / 32) * 2;
            uint8_t* ds = st + (size_t)NM * R * cb + (size_t)i * R * gs * 2;
            uint8_t* dm = st + (size_t)NM * R * cb + (size_t)NM * R * gs * 2 + (size_t)i * R * gs * 2;
            if (klen == job.K) {
              bulk_g2s(ds, sc, (uint32_t)(nr * gs * 2), &full[slot]);
              bulk_g2s(dm, mn, (uint32_t)(nr * gs * 2), &full[slot]);
            } else {
              for (int r = 0; r < nr; ++r) {
                bulk_g2s(ds + r * gs * 2, sc + (size_t)r * row_groups * 2, gs * 2, &full[slot]);
                bulk_g2s(dm + r * gs * 2, mn + (size_t)r * row_groups * 2, gs * 2, &full[slot]);
              }
            }
          }
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int nthreads = NC * 32;
  const uint16_t* src = job.shared ? a.x_s : a.x;
  const int ld = job.shared ? job.K : a.ld_x;
  int s = 0;
  bool dead = false;
  for (int tb = 0; tb < job.ntok; tb += a.stage_tokens) {
    const int tn = min(a.stage_tokens, job.ntok - tb);
    consumer_sync(nthreads);
    // Stage token rows tb..tb+tn (K slice) as position-scaled fp32; zero pad rows.
    const int per_row = klen / 8;
    for (int i = threadIdx.x; i < tok_rows * per_row; i += nthreads) {
      const int r = i / per_row;
      const int kk = (i - r * per_row) * 8;
      float f[8];
      if (r < tn) {
        const int row = job.gather ? a.perm[job.slot0 + tb + r] / a.topk : job.slot0 + tb + r;
        const uint4 v = *reinterpret_cast<const uint4*>(src + (size_t)row * ld + k0 + kk);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          f[2 * j] = __uint_as_float(w[j] << 16) * C::pos_scale(kk + 2 * j);
          f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u) * C::pos_scale(kk + 2 * j + 1);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) f[j] = 0.f;
      }
      const int c = kk / C::kChunk, o = kk - c * C::kChunk;
      float* dst = xs + r * tok_stride + c * C::kStride + o;
      *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
      *reinterpret_cast<float4*>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
    }
    if (kInt4) {
      const int gsd = gs > 0 ? gs : 1;
      for (int i = threadIdx.x; i < tok_rows * gs; i += nthreads) {
        const int r = i / gsd, g = i - r * gsd;
        float sum = 0.f;
        if (r < tn) {
          const int row = job.gather ? a.perm[job.slot0 + tb + r] / a.topk : job.slot0 + tb + r;
          const uint16_t* p = src + (size_t)row * ld + k0 + g * 32;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint4 v = *reinterpret_cast<const uint4*>(p + 8 * q);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) sum += __uint_as_float(w[j] << 16) + __uint_as_float(w[j] & 0xFFFF0000u);
          }
        }
        xsum[r * gs + g] = sum;
      }
    }
    consumer_sync(nthreads);

    for (int rs = 0; rs < row_stages; ++rs, ++s) {
      const int slot = s % S, use = s / S;
      const int n = r0 + rs * R + warp;
      float row_scale[NM];
      if (!kInt4 && n < r1) {
#pragma unroll
        for (int i = 0; i < NM; ++i) row_scale[i] = __half2float(__ldg(job.m[i].scale + n));
      }
      // After a timed-out wait (a fault already recorded) the warp stops
      // computing but still takes part in every barrier below.
      if (!dead && !mbar_wait(&full[slot], use & 1)) dead = true;
      if (!dead && n < r1) {
        const uint8_t* st = stage0 + (size_t)slot * stage_bytes;
        const uint8_t* codes[NM];
        const __half* scl[NM];
        const __half* mns[NM];
#pragma unroll
        for (int i = 0; i < NM; ++i) {
          codes[i] = st + ((size_t)i * R + warp) * cb;
          scl[i] = reinterpret_cast<const __half*>(st + (size_t)NM * R * cb) + ((size_t)i * R + warp) * gs;
          mns[i] = reinterpret_cast<const __half*>(st + (size_t)NM * R * cb + (size_t)NM * R * gs * 2) +
                   ((size_t)i * R + warp) * gs;
        }
        for (int tc = 0; tc < tn; tc += MT) {
          float acc[NM][MT];
#pragma unroll
          for (int i = 0; i < NM; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[i][t] = 0.f;
          const float* xb = xs + tc * tok_stride;
          for (int c = lane; c < nch; c += 32) {
            uint4 wv[NM];
            float sc[NM], mn[NM];
#pragma unroll
            for (int i = 0; i < NM; ++i) {
              wv[i] = *reinterpret_cast<const uint4*>(codes[i] + c * 16);
              if (kInt4) {
                sc[i] = __half2float(scl[i][c]);
                mn[i] = __half2float(mns[i][c]);
              }
            }
            float2 p[NM][MT];
#pragma unroll
            for (int i = 0; i < NM; ++i)
#pragma unroll
              for (int t = 0; t < MT; ++t) p[i][t] = make_float2(0.f, 0.f);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              float2 cf[NM][4];
#pragma unroll
              for (int i = 0; i < NM; ++i) {
                const uint32_t w = q == 0 ? wv[i].x : q == 1 ? wv[i].y : q == 2 ? wv[i].z : wv[i].w;
                C::word(w, cf[i]);
              }
#pragma unroll
              for (int t = 0; t < MT; ++t) {
                const float* xp = xb + t * tok_stride + c * C::kStride + q * 2 * C::kFloat2;
                const float4 xa = *reinterpret_cast<const float4*>(xp);
                float4 xc = make_float4(0.f, 0.f, 0.f, 0.f);
                if (C::kFloat2 == 4) xc = *reinterpret_cast<const float4*>(xp + 4);
#pragma unroll
                for (int i = 0; i < NM; ++i) {
                  p[i][t] = __ffma2_rn(cf[i][0], make_float2(xa.x, xa.y), p[i][t]);
                  p[i][t] = __ffma2_rn(cf[i][1], make_float2(xa.z, xa.w), p[i][t]);
                  if (C::kFloat2 == 4) {
                    p[i][t] = __ffma2_rn(cf[i][2], make_float2(xc.x, xc.y), p[i][t]);
                    p[i][t] = __ffma2_rn(cf[i][3], make_float2(xc.z, xc.w), p[i][t]);
                  }
                }
              }
            }
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              const float X = kInt4 ? xsum[(tc + t) * gs + c] : 0.f;
#pragma unroll
              for (int i = 0; i < NM; ++i) {
                const float P = p[i][t].x + p[i][t].y;
                acc[i][t] = kInt4 ? fmaf(sc[i], P, fmaf(mn[i], X, acc[i][t])) : acc[i][t] + P;
              }
            }
          }
          // epilogue
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            float v[NM];
#pragma unroll
            for (int i = 0; i < NM; ++i) {
              v[i] = warp_sum(acc[i][t]);
              if (!kInt4) v[i] *= row_scale[i];
            }
            const int tok = tb + tc + t;
            if (lane == 0 && tok < tn + tb) {
              const int slot_out = job.slot0 + tok;
              if (NM == 2) {
                uint16_t* out = job.shared ? a.out_act_s : a.out_act;
                out[(size_t)slot_out * job.N + n] = float_to_bf16_bits(gated_act(v[0], v[NM - 1], a.act));
              } else {
                float* d = job.shared ? a.out_d_s : a.out_d;
                const int nslots = job.shared ? a.M : a.slots;
                d[((size_t)blockIdx.y * nslots + slot_out) * job.N + n] = v[0];
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  }
}

template <int FMT, int MT, int NM, int NC>
cudaError_t launch_one(const TmaGemvArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
  auto kern = k_gemv_tma<FMT, MT, NM, NC>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, 32 * (NC + 1), smem, s>>>(a);
  return cudaGetLastError();
}

template <int FMT, int NM>
cudaError_t launch_fmt(const TmaGemvArgs& a, int mt, dim3 grid, size_t smem, cudaStream_t s) {
  return mt == 1 ? launch_one<FMT, 1, NM, kTmaConsumers>(a, grid, smem, s)
                 : launch_one<FMT, 2, NM, kTmaConsumers>(a, grid, smem, s);
}

}  // namespace

size_t tma_gemv_smem(int fmt, int nm, int klen, int stage_tokens, int mt, int stages) {
  const bool i4 = fmt == FMT_INT4_G32;
  const int chunk = i4 ? 32 : 16, stride = i4 ? 36 : 20;
  const int gs = i4 ? klen / 32 : 0;
  const int tok_rows = (stage_tokens + mt - 1) / mt * mt;
  const size_t x_bytes = ((size_t)tok_rows * ((klen / chunk) * stride + gs) * 4 + 127) / 128 * 128;
  const size_t stage_bytes = (size_t)nm * kTmaConsumers * ((i4 ? klen / 2 : klen) + 4 * gs);
  return 128 + x_bytes + stage_bytes * stages;
}

size_t tma_gemv_stage_bytes(int fmt, int nm, int klen) {
  const bool i4 = fmt == FMT_INT4_G32;
  return (size_t)nm * kTmaConsumers * ((i4 ? klen / 2 : klen) + 4 * (i4 ? klen / 32 : 0));
}

cudaError_t launch_tma_gemv(const TmaGemvArgs& a, int nm, int mt, int splits, int jobs, cudaStream_t s) {
  const size_t smem = tma_gemv_smem(a.fmt, nm, a.ks_len, a.stage_tokens, mt, a.stages);
  const dim3 grid(a.ctas_per_job, splits, jobs);
  if (a.fmt == FMT_INT4_G32)
    return nm == 2 ? launch_fmt<FMT_INT4_G32, 2>(a, mt, grid, smem, s) : launch_fmt<FMT_INT4_G32, 1>(a, mt, grid, smem, s);
  return nm == 2 ? launch_fmt<FMT_INT8_ROW, 2>(a, mt, grid, smem, s) : launch_fmt<FMT_INT8_ROW, 1>(a, mt, grid, smem, s);
}

unsigned int tma_gemv_fault_flags(bool clear) {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_fault_flags, sizeof(v));
  if (clear && v) {
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_fault_flags, &z, sizeof(z));
  }
  return v;
}

}  // namespace moeffn
