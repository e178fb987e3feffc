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
#include "gemv_math.cuh"
#include "sync.cuh"
#include "tmap.cuh"
#include "launch.cuh"

namespace moeffn {

namespace {

struct Job {
  QW m[2];
  int N, K, ntok, slot0, expert;
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
    j.expert = e;
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

// NC consumer warps per group, G groups: group g takes the stages s with
// s % G == g, one row of the stage per warp (R = NC rows per stage). The ring
// depth S is a multiple of G, so every slot is waited on by one group only,
// in stage order: a waiter is never two phases ahead of a slot's barriers
// (whose phase parity would then alias the previous use).
//
// NM = 2: gate and up, R rows of each per stage. PR (row pairs, a single
// matrix: the down projection): a stage holds 2R consecutive rows of one
// matrix in the same layout, and each warp computes rows n and n + R, so that
// the activations it loads from shared memory serve two rows.
template <int FMT, int MT, int NM, int NC, int G, bool PR = false>
__global__ void __launch_bounds__(32 * (NC * G + 1), 1) k_gemv_tma(const __grid_constant__ TmaGemvArgs a) {
  static_assert(!PR || NM == 2, "row pairs use the two-matrix stage layout");
  using C = Codes<FMT>;
  constexpr bool kInt4 = (FMT == FMT_INT4_G32);
  constexpr bool kQ4K = (FMT == FMT_Q4K);
  constexpr bool kAffine = kInt4 || kQ4K;   // a min term: staged chunk sums needed
  constexpr int R = NC;  // rows per stage
  extern __shared__ __align__(128) uint8_t smem[];

  // A dense job's producer reads only weights, which no kernel writes, so it
  // starts streaming while the previous kernel in the stream finishes; the
  // consumers (activations in, outputs out) and grouped jobs (whose expert
  // lists the routing kernels write) wait for it first.
  const bool early = a.offsets == nullptr;
  if (!early) pdl_wait();
  if (a.stages < G || a.stages % G != 0 || a.stages > 8) {   // ring depth the host must not choose
    if (threadIdx.x == 0) atomicOr(&g_fault_flags, 2u);
    return;
  }
  const Job job = decode_job(a);
  if (!job.valid || job.ntok == 0) return;
  const int k0 = blockIdx.y * a.ks_len;
  if (k0 >= job.K) return;
  const int klen = min(a.ks_len, job.K - k0);
  constexpr int RS = PR ? 2 * R : R;   // rows per stage
  const int rpc = ((job.N + a.ctas_per_job - 1) / a.ctas_per_job + RS - 1) / RS * RS;
  const int r0 = blockIdx.x * rpc;
  const int r1 = min(job.N, r0 + rpc);
  if (r0 >= r1) return;
  // A job split along K loads boxes through its tensor maps; an unsplit job
  // copies whole (contiguous) rows.
  const bool maps = a.use_maps != 0 && job.K > a.ks_len;
  const QWMaps* jm = nullptr;
  if (maps) jm = a.offsets == nullptr ? &a.dmap : (job.shared ? a.maps_s : a.maps + job.expert);

  // ---- shared memory carve ------------------------------------------------
  // Stage rows are `cs` code bytes and `gst` groups apart: the full box width
  // (ks_len) with tensor maps, the slice itself with 1-D copies.
  const int S = a.stages;
  const int wid = maps ? a.ks_len : klen;
  const int cs = kInt4 ? wid / 2 : kQ4K ? wid / Q4K::kBlock * Q4K::kBytes : wid;
  const int gst = kInt4 ? wid / 32 : 0;
  const int nch = klen / C::kChunk;
  const int tok_stride = nch * C::kStageBytes;   // bytes of staged int16 per token
  const int tok_rows = (a.stage_tokens + MT - 1) / MT * MT;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + S;
  uint8_t* xi = smem + 128;                                         // [tok_rows][nch] chunks
  float* xf = reinterpret_cast<float*>(xi + (size_t)tok_rows * tok_stride);  // [tok_rows][nch] factors
  float* xsum = xf + (size_t)tok_rows * nch;                        // [tok_rows][nch] (INT4, Q4_K)
  const size_t x_bytes = ((size_t)tok_rows * (tok_stride + 4 * nch + (kAffine ? 4 * nch : 0)) + 127) / 128 * 128;
  // then the input norm's scratch (gemv_norm_bytes)
  uint8_t* stage0 = smem + 128 + x_bytes + gemv_norm_bytes(NC * G);
  const size_t stage_bytes = (size_t)NM * R * (cs + 4 * gst);
  // within a stage: codes [NM][R][cs], scales [NM][R][gst], mins [NM][R][gst]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], NC);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int row_stages = (r1 - r0 + RS - 1) / RS;
  const int tok_blocks = (job.ntok + a.stage_tokens - 1) / a.stage_tokens;
  const int total = row_stages * tok_blocks;
  const int row_bytes = kInt4 ? job.K / 2 : kQ4K ? job.K / Q4K::kBlock * Q4K::kBytes : job.K;
  const int row_groups = job.K / 32;

  // The next kernel in the stream may be scheduled now; it waits for this
  // grid's completion before reading what this grid writes.
  pdl_launch_dependents();
  const unsigned long long wait_ns = a.wait_ns != 0 ? a.wait_ns : kWaitLimitNs;
  if (warp == NC * G) {
    // ---------------- producer ----------------
    if (lane == 0) {
      for (int s = 0; s < total; ++s) {
        const int slot = s % S, use = s / S;
        if (a.inject_stop > 0 && s >= a.inject_stop - 1) break;   // injected producer failure (tests)
        if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1, wait_ns)) break;
        const int n0 = r0 + (s % row_stages) * RS;
        const int nr = min(R, r1 - n0);
        uint8_t* st = stage0 + (size_t)slot * stage_bytes;
        uint8_t* dsc = st + (size_t)NM * R * cs;
        uint8_t* dmn = dsc + (size_t)NM * R * gst * 2;
        if (maps) {
          // Whole boxes: rows past the end of the matrix arrive as zeros.
          mbar_arrive_expect_tx(&full[slot], (uint32_t)stage_bytes);
#pragma unroll
          for (int i = 0; i < NM; ++i) {
            // x in 8-byte elements: 16 INT4 codes, 8 INT8 codes, or 18 per Q4_K block
            const QWMaps& mp = jm[PR ? 0 : i];
            const int ny = n0 + (PR ? i * R : 0);   // rows past the end arrive as zeros
            tma_load_2d(st + (size_t)i * R * cs, &mp.codes, kInt4 ? k0 / 16 : kQ4K ? k0 / Q4K::kBlock * 18 : k0 / 8,
                        ny, &full[slot]);
            if (kInt4) {
              tma_load_2d(dsc + (size_t)i * R * gst * 2, &mp.scale, k0 / 32, ny, &full[slot]);
              tma_load_2d(dmn + (size_t)i * R * gst * 2, &mp.mn, k0 / 32, ny, &full[slot]);
            }
          }
        } else {
          // Whole rows are contiguous: one copy per array for the stage.
          const int nr1 = PR ? max(0, min(R, r1 - (n0 + R))) : nr;   // rows of the second half
          mbar_arrive_expect_tx(&full[slot], (uint32_t)((nr + (NM == 2 ? nr1 : 0)) * (cs + 4 * gst)));
#pragma unroll
          for (int i = 0; i < NM; ++i) {
            const QW& mq = job.m[PR ? 0 : i];
            const int ni = n0 + (PR ? i * R : 0), cnt = i == 0 ? nr : nr1;
            if (cnt > 0) {
              bulk_g2s(st + (size_t)i * R * cs, mq.q + (size_t)ni * row_bytes, (uint32_t)(cnt * cs), &full[slot]);
              if (kInt4) {
                const size_t go = (size_t)ni * row_groups * 2;
                bulk_g2s(dsc + (size_t)i * R * gst * 2, reinterpret_cast<const uint8_t*>(mq.scale) + go,
                         (uint32_t)(cnt * gst * 2), &full[slot]);
                bulk_g2s(dmn + (size_t)i * R * gst * 2, reinterpret_cast<const uint8_t*>(mq.mn) + go,
                         (uint32_t)(cnt * gst * 2), &full[slot]);
              }
            }
          }
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  if (early) pdl_wait();
  const int nthreads = NC * G * 32;
  if (a.zero_cnt != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int i = threadIdx.x; i < a.zero_n; i += nthreads) a.zero_cnt[i] = 0;
  const int grp = warp / NC, wr = warp - grp * NC;  // group, row of the stage
  // Shared memory of the input-norm pass: [tok_rows] inverse RMS values, then
  // [tok_rows][consumer warps] partial sums of squares.
  float* norm_buf = reinterpret_cast<float*>(smem + 128 + x_bytes);
  const uint16_t* src = job.shared ? a.x_s : a.x;
  const int ld = job.shared ? job.K : a.ld_x;
  bool dead = false;
  for (int tb = 0, tbi = 0; tb < job.ntok; tb += a.stage_tokens, ++tbi) {
    const int tn = min(a.stage_tokens, job.ntok - tb);
    consumer_sync(nthreads);
    // Input norm folded in (dense gate/up: the job's whole row is this CTA's
    // K range): inv_rms of every staged token row, from per-warp sums of
    // squares added in warp order.
    const bool norm = a.norm_w != nullptr;
    float* inv_rms = norm_buf;                        // [tok_rows], then [tok_rows][warps] partial sums
    if (norm) {
      const int nw = nthreads / 32;
      float* ssp = inv_rms + tok_rows;
      for (int r = 0; r < tn; ++r) {
        float ss = row_sumsq_part(src + (size_t)(job.slot0 + tb + r) * ld, job.K, threadIdx.x, nthreads);
        ss = warp_sum(ss);
        if (lane == 0) ssp[r * nw + warp] = ss;
      }
      consumer_sync(nthreads);
      if (threadIdx.x < tn) {
        float ss = 0.f;
        for (int w = 0; w < nw; ++w) ss += ssp[threadIdx.x * nw + w];
        inv_rms[threadIdx.x] = inv_rms_of(ss, job.K, a.eps);
      }
      consumer_sync(nthreads);
    }
    // Stage token rows tb..tb+tn (K slice) chunk by chunk: int16 fixed point,
    // the chunk's power-of-two factor and (INT4) its plain sum; zero pad rows.
    for (int i = threadIdx.x; i < tok_rows * nch; i += nthreads) {
      const int r = i / nch, c = i - r * nch;
      const uint16_t* p = nullptr;
      if (r < tn) {
        const int row = job.gather ? a.perm[job.slot0 + tb + r] / a.topk : job.slot0 + tb + r;
        p = src + (size_t)row * ld + k0 + c * C::kChunk;
      }
      stage_chunk<FMT>(p, xi + r * tok_stride + c * C::kStageBytes, &xf[r * nch + c], &xsum[r * nch + c],
                       (norm && p != nullptr) ? a.norm_w + k0 + c * C::kChunk : nullptr,
                       (norm && p != nullptr) ? inv_rms[r] : 0.f);
    }
    consumer_sync(nthreads);

    for (int rs = grp; rs < row_stages; rs += G) {
      const int s = tbi * row_stages + rs;
      const int slot = s % S, use = s / S;
      const int n = r0 + rs * RS + wr;
      float row_scale[NM];
      if (FMT == FMT_INT8_ROW && n < r1) {
#pragma unroll
        for (int i = 0; i < NM; ++i) {
          const int ni = n + (PR ? i * R : 0);
          row_scale[i] = ni < r1 ? __half2float(__ldg(job.m[PR ? 0 : i].scale + ni)) : 0.f;
        }
      }
      // After a timed-out wait (a fault already recorded) the warp stops
      // computing but still takes part in every barrier below.
      if (!dead && !mbar_wait(&full[slot], use & 1, wait_ns)) dead = true;
      if (!dead && n < r1) {
        // 32-bit byte offsets from the stage start (shared memory).
        const uint8_t* st = stage0 + slot * (int)stage_bytes;
        int o_code[NM], o_sc[NM];
#pragma unroll
        for (int i = 0; i < NM; ++i) {
          o_code[i] = (i * R + wr) * cs + lane * 16;
          o_sc[i] = NM * R * cs + ((i * R + wr) * gst + lane) * 2;
        }
        const int mn_off = NM * R * gst * 2;   // mins follow the scales
        for (int tc = 0; tc < tn; tc += MT) {
          float acc[NM][MT];
#pragma unroll
          for (int i = 0; i < NM; ++i)
#pragma unroll
            for (int t = 0; t < MT; ++t) acc[i][t] = 0.f;
          if (kQ4K) {
            // A lane takes code runs u = lane, lane + 32, ...: run u % 4 of
            // block u / 4 (32 code bytes, two sub-blocks), whose scales and
            // mins come from the block's 16-byte header.
            const int nu = klen / 64;
            for (int u = lane; u < nu; u += 32) {
              const int bo = (u >> 2) * Q4K::kBytes;
              const int ox = tc * tok_stride + 2 * u * C::kStageBytes;
              const int of = tc * nch + 2 * u;
              uint4 c0[NM], c1[NM];
#pragma unroll
              for (int i = 0; i < NM; ++i) {
                const uint8_t* rb = st + (i * R + wr) * cs + bo + 16 + 32 * (u & 3);
                c0[i] = *reinterpret_cast<const uint4*>(rb);
                c1[i] = *reinterpret_cast<const uint4*>(rb + 16);
              }
              int pl[NM][MT], ph[NM][MT];
#pragma unroll
              for (int t = 0; t < MT; ++t) {
                const uint8_t* xl = xi + ox + t * tok_stride;
                const uint8_t* xh = xl + C::kStageBytes;
#pragma unroll
                for (int i = 0; i < NM; ++i) pl[i][t] = ph[i][t] = 0;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  const uint4 a = *reinterpret_cast<const uint4*>(xl + 16 * h);
                  const uint4 b = *reinterpret_cast<const uint4*>(xh + 16 * h);
#pragma unroll
                  for (int i = 0; i < NM; ++i) {
                    const uint4& cw = h < 2 ? c0[i] : c1[i];
                    const uint32_t w0 = (h & 1) ? cw.z : cw.x, w1 = (h & 1) ? cw.w : cw.y;
                    Codes<FMT_Q4K>::dot_words(w0, w1, a, b, pl[i][t], ph[i][t]);
                  }
                }
              }
#pragma unroll
              for (int i = 0; i < NM; ++i) {
                const uint4 hdr = *reinterpret_cast<const uint4*>(st + (i * R + wr) * cs + bo);
                float sl, ml, sh, mh;
                Q4K::scale_min(hdr, 2 * (u & 3), sl, ml);
                Q4K::scale_min(hdr, 2 * (u & 3) + 1, sh, mh);
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                  const float fl = xf[of + t * nch], fh = xf[of + 1 + t * nch];
                  const float Xl = xsum[of + t * nch], Xh = xsum[of + 1 + t * nch];
                  // sum over both sub-blocks of (d sc q - dmin m) x
                  float v = fmaf(ml, Xl, acc[i][t]);
                  v = fmaf(sl * fl, (float)pl[i][t], v);
                  v = fmaf(mh, Xh, v);
                  acc[i][t] = fmaf(sh * fh, (float)ph[i][t], v);
                }
              }
            }
          } else {
          int ox = tc * tok_stride + lane * C::kStageBytes;   // staged activations
          int of = tc * nch + lane;                            // factors / sums
          int oc = 0, og = 0;                                  // code / scale advance
          for (int c = lane; c < nch; c += 32, ox += 32 * C::kStageBytes, of += 32, oc += 512, og += 64) {
            uint4 wv[NM];
            float sc[NM], mn[NM];
#pragma unroll
            for (int i = 0; i < NM; ++i) {
              wv[i] = *reinterpret_cast<const uint4*>(st + o_code[i] + oc);
              if (kInt4) {
                sc[i] = __half2float(*reinterpret_cast<const __half*>(st + o_sc[i] + og));
                mn[i] = __half2float(*reinterpret_cast<const __half*>(st + o_sc[i] + og + mn_off));
              }
            }
            int p0[NM][MT], p1[NM][MT];
#pragma unroll
            for (int i = 0; i < NM; ++i)
#pragma unroll
              for (int t = 0; t < MT; ++t) p0[i][t] = p1[i][t] = 0;
            if (kInt4) {
#pragma unroll
              for (int q = 0; q < 4; ++q) {
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                  const uint4 x4 = *reinterpret_cast<const uint4*>(xi + ox + t * tok_stride + q * 16);
#pragma unroll
                  for (int i = 0; i < NM; ++i) {
                    const uint32_t w = q == 0 ? wv[i].x : q == 1 ? wv[i].y : q == 2 ? wv[i].z : wv[i].w;
                    Codes<FMT_INT4_G32>::dot_word(w, x4, p0[i][t], p1[i][t]);
                  }
                }
              }
            } else {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
#pragma unroll
                for (int t = 0; t < MT; ++t) {
                  const uint4 x4 = *reinterpret_cast<const uint4*>(xi + ox + t * tok_stride + h * 16);
#pragma unroll
                  for (int i = 0; i < NM; ++i) {
                    const uint32_t w0 = h == 0 ? wv[i].x : wv[i].z, w1 = h == 0 ? wv[i].y : wv[i].w;
                    Codes<FMT_INT8_ROW>::dot_word(w0, w1, x4, p0[i][t], p1[i][t]);
                  }
                }
              }
            }
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              const float f = xf[of + t * nch];
              const float X = kInt4 ? xsum[of + t * nch] : 0.f;
#pragma unroll
              for (int i = 0; i < NM; ++i) {
                const float P = (float)(p0[i][t] + p1[i][t]);   // exact below 2^24
                // sum_k (q_k s + m) x_k = s * 2^(e-14) * sum_k q_k xi_k + m * sum_k x_k
                acc[i][t] = kInt4 ? fmaf(sc[i] * f, P, fmaf(mn[i], X, acc[i][t])) : fmaf(f, P, acc[i][t]);
              }
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
              if (FMT == FMT_INT8_ROW) v[i] *= row_scale[i];
            }
            const int tok = tb + tc + t;
            if (lane == 0 && tok < tn + tb) {
              const int slot_out = job.slot0 + tok;
              if (NM == 2 && !PR) {
                uint16_t* out = job.shared ? a.out_act_s : a.out_act;
                out[(size_t)slot_out * job.N + n] = float_to_bf16_bits(gated_act(v[0], v[NM - 1], a.act));
              } else {
                float* d = job.shared ? a.out_d_s : a.out_d;
                const int nslots = job.shared ? a.M : a.slots;
#pragma unroll
                for (int i = 0; i < NM; ++i) {
                  const int ni = n + (PR ? i * R : 0);
                  if (i == 0 || ni < r1) d[((size_t)blockIdx.y * nslots + slot_out) * job.N + ni] = v[i];
                }
              }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }
  }

  if (a.res != nullptr) {
    // Residual tail folded in (dense down projection): the last of the K
    // splits to finish this CTA's row range adds the splits' partial sums in
    // split order, rounds to bf16 and adds the result to the residual, as the
    // tail kernel would.
    __threadfence();
    consumer_sync(nthreads);
    int* last = reinterpret_cast<int*>(xi);   // staged activations are no longer read
    if (threadIdx.x == 0) {
      const int old = atomicAdd(&a.tile_cnt[blockIdx.x], 1);
      *last = old == (int)gridDim.y - 1;
      if (*last) a.tile_cnt[blockIdx.x] = 0;  // ready for the next call
    }
    consumer_sync(nthreads);
    if (*last) {
      __threadfence();
      const int nr = r1 - r0;
      const size_t stride = (size_t)a.slots * job.N;
      for (int i = threadIdx.x; i < nr * job.ntok; i += nthreads) {
        const int t = i / nr, n = r0 + (i - t * nr);
        const size_t o = (size_t)t * job.N + n;
        float h = 0.f;
        for (int sp = 0; sp < (int)gridDim.y; ++sp) h += __ldcg(a.out_d + sp * stride + o);
        a.res[o] = float_to_bf16_bits(bf16_bits_to_float(a.res[o]) + round_bf16(h));
      }
    }
  }
}

// PR: one matrix in row pairs (the two-matrix stage layout); else gate + up.
template <int FMT, int MT, bool PR>
cudaError_t launch_one(const TmaGemvArgs& a, dim3 grid, size_t smem, cudaStream_t s) {
  auto kern = k_gemv_tma<FMT, MT, 2, kTmaConsumers, kTmaGroups, PR>;
  static bool opted[64] = {};   // opted in to the 227 KB maximum
  const cudaError_t e = opt_in_smem(kern, 227 * 1024, opted);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, dim3(32 * (kTmaConsumers * kTmaGroups + 1)), smem, s, a);
}

template <int FMT, bool PR>
cudaError_t launch_fmt(const TmaGemvArgs& a, int mt, dim3 grid, size_t smem, cudaStream_t s) {
  return mt == 1 ? launch_one<FMT, 1, PR>(a, grid, smem, s) : launch_one<FMT, 2, PR>(a, grid, smem, s);
}

template <bool PR>
cudaError_t launch_any(const TmaGemvArgs& a, int mt, dim3 grid, size_t smem, cudaStream_t s) {
  if (a.fmt == FMT_INT4_G32) return launch_fmt<FMT_INT4_G32, PR>(a, mt, grid, smem, s);
  if (a.fmt == FMT_Q4K) return launch_fmt<FMT_Q4K, PR>(a, mt, grid, smem, s);
  return launch_fmt<FMT_INT8_ROW, PR>(a, mt, grid, smem, s);
}

}  // namespace

size_t tma_gemv_stage_bytes(int fmt, int nm, int klen);

size_t tma_gemv_smem(int fmt, int nm, int klen, int stage_tokens, int mt, int stages) {
  const bool affine = fmt == FMT_INT4_G32 || fmt == FMT_Q4K;   // staged chunk sums
  const size_t red = gemv_norm_bytes(kTmaConsumers * kTmaGroups);
  const int nch = klen / (fmt == FMT_INT8_ROW ? 16 : 32);
  const int cbytes = fmt == FMT_INT8_ROW ? Codes<FMT_INT8_ROW>::kStageBytes : Codes<FMT_INT4_G32>::kStageBytes;
  const int tok_rows = (stage_tokens + mt - 1) / mt * mt;
  const size_t x_bytes =
      ((size_t)tok_rows * ((size_t)nch * cbytes + 4 * nch + (affine ? 4 * nch : 0)) + 127) / 128 * 128;
  return 128 + x_bytes + red + tma_gemv_stage_bytes(fmt, nm, klen) * stages;
}

size_t tma_gemv_stage_bytes(int fmt, int nm, int klen) {
  size_t row;
  if (fmt == FMT_INT4_G32) row = klen / 2 + 4 * (klen / 32);   // codes, scales, mins
  else if (fmt == FMT_Q4K) row = (size_t)klen / Q4K::kBlock * Q4K::kBytes;
  else row = klen;
  return (size_t)nm * kTmaConsumers * row;
}

cudaError_t launch_tma_gemv(const TmaGemvArgs& a, int nm, int mt, int splits, int jobs, cudaStream_t s) {
  const dim3 grid(a.ctas_per_job, splits, jobs);
  const size_t smem = tma_gemv_smem(a.fmt, 2, a.ks_len, a.stage_tokens, mt, a.stages);
  return nm == 1 ? launch_any<true>(a, mt, grid, smem, s) : launch_any<false>(a, mt, grid, smem, s);
}

cudaError_t encode_qw_maps(QWMaps* m, int fmt, const QW& w, int N, int K, int ks_len) {
  const int R = kTmaConsumers;
  cudaError_t e;
  if (fmt == FMT_INT4_G32) {
    e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT64, w.q, K / 16, N, K / 2, ks_len / 16, R);
    if (e != cudaSuccess) return e;
    e = encode_tmap_2d(&m->scale, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.scale, K / 32, N, K / 16, ks_len / 32, R);
    if (e != cudaSuccess) return e;
    return encode_tmap_2d(&m->mn, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.mn, K / 32, N, K / 16, ks_len / 32, R);
  }
  if (fmt == FMT_Q4K) {   // 18 eight-byte elements per block; the boxes hold whole blocks
    e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT64, w.q, K / Q4K::kBlock * 18, N,
                       (size_t)K / Q4K::kBlock * Q4K::kBytes, ks_len / Q4K::kBlock * 18, R);
    m->scale = m->codes;
    m->mn = m->codes;
    return e;
  }
  e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT64, w.q, K / 8, N, K, ks_len / 8, R);
  m->scale = m->codes;
  m->mn = m->codes;
  return e;
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
