// Whole dense FFN for one or two token rows as a single weight stream.
//
// At decode sizes the FFN reads every weight once and does 1-2 multiply-adds
// per weight, so its time is the time to stream the weights from HBM. Run as
// separate GEMV launches, each launch pays its own pipeline fill (the first
// stages of every SM arrive together) and a ragged end, which at 20 us per
// launch costs a third of the bandwidth. Here one persistent CTA per SM
// streams its rows of gate/up (phase A) and then its rows of down (phase B)
// through one ring of shared-memory stages without a break:
//
//  warp 16     producer: 2-D TMA boxes of [rows][K chunk] of the codes (and
//              INT4 scales and mins) into the ring, phase A then phase B;
//  warps 0-15  consumers: phase A takes blocks of 8 gate/up row pairs, two
//              warps per row, and writes h = bf16(act(gate.x) * up.x) to a
//              workspace row; after a grid barrier (all of h written) phase B
//              takes blocks of 4 down rows, four warps per row, each row's full
//              dot product in one CTA, and writes the layer's output directly:
//              residual + bf16(y) (llama), or y for the post-FFN RMSNorm,
//              applied after a second grid barrier (Gemma shared expert).
//
// The producer never waits on the grid barrier, so phase B's first stages are
// in shared memory when the barrier opens. Dot products use the GEMV's int16
// fixed-point activations and DP2A (gemv_math.cuh).
//
// The grid barrier spins on a device counter: the launch is cooperative (all
// CTAs resident), and a wait that passes about a second records fault bit 2
// and lets the CTA go on (its outputs are then not to be trusted).
#include "ffn_stream.cuh"

#include <algorithm>

#include "gemv_math.cuh"
#include "sync.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace moeffn {

namespace {

constexpr int kConsumerWarps = 16;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kRowsA = 8, kWarpsPerRowA = 2;   // phase A: gate/up row pairs per stage
constexpr int kRowsB = 4, kWarpsPerRowB = 4;   // phase B: down rows per stage

// Grid barriers: [2 * i] arrivals, counted up forever (a barrier is complete
// when the count reaches a multiple of the grid size), [2 * i + 1] generation,
// advanced by the arrival that completes it.
__device__ unsigned long long g_grid_bar[4] = {0, 0, 0, 0};

__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ unsigned long long add_acq_rel(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.acq_rel.gpu.global.add.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}
__device__ __forceinline__ void add_release(unsigned long long* p, unsigned long long v) {
  asm volatile("red.release.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// All consumer threads of every CTA call this; thread ct == 0 takes part for
// its CTA (the CTA barrier before it orders the CTA's writes before its
// release). Returns false (fault recorded) if the wait ran out.
__device__ bool grid_barrier(int idx, int ct) {
  named_sync(1, 32 * kConsumerWarps);
  __shared__ int ok_s;
  if (ct == 0) {
    unsigned long long* count = &g_grid_bar[2 * idx];
    unsigned long long* gen = &g_grid_bar[2 * idx + 1];
    const unsigned long long g = ld_acquire(gen);
    const unsigned long long prev = add_acq_rel(count, 1ull);
    int ok = 1;
    if ((prev + 1) % gridDim.x == 0) {
      add_release(gen, 1ull);
    } else {
      const unsigned long long t0 = global_ns();
      while (ld_acquire(gen) == g) {
        if (global_ns() - t0 > kWaitLimitNs) {
          atomicOr(&g_fault_flags, 4u);
          ok = 0;
          break;
        }
      }
    }
    ok_s = ok;
  }
  named_sync(1, 32 * kConsumerWarps);
  return ok_s != 0;
}

// Stage geometry of one phase: R rows x kc codes per stage, in boxes of `box`
// codes along K (nbox per stage), NM matrices.
struct Geo {
  int R, NM, kc, box, nbox;
  int code_bytes;   // per box row
  int sc_bytes;     // per box row (INT4 scales; mins the same)
  int off_sc, off_mn, bytes;
};

template <int FMT>
__device__ __forceinline__ Geo make_geo(int R, int NM, int kc, int box) {
  Geo g;
  g.R = R; g.NM = NM; g.kc = kc; g.box = box; g.nbox = kc / box;
  g.code_bytes = FMT == FMT_INT4_G32 ? box / 2 : box;
  g.sc_bytes = FMT == FMT_INT4_G32 ? box / 16 : 0;
  const int boxes = NM * g.nbox;
  g.off_sc = boxes * R * g.code_bytes;
  g.off_mn = g.off_sc + boxes * R * g.sc_bytes;
  g.bytes = g.off_mn + boxes * R * g.sc_bytes;
  return g;
}

// Issues the TMA boxes of one stage (rows row0.., K from k0) into dst.
template <int FMT>
__device__ __forceinline__ void load_stage(const Geo& g, const QWMaps* maps, uint8_t* dst, int row0, int k0,
                                           uint64_t* bar) {
  mbar_arrive_expect_tx(bar, (uint32_t)g.bytes);
  for (int i = 0; i < g.NM; ++i) {
    for (int bx = 0; bx < g.nbox; ++bx) {
      const int kb = k0 + bx * g.box;
      const int b = i * g.nbox + bx;
      tma_load_2d(dst + b * g.R * g.code_bytes, &maps[i].codes, FMT == FMT_INT4_G32 ? kb / 16 : kb / 8, row0, bar);
      if (FMT == FMT_INT4_G32) {
        tma_load_2d(dst + g.off_sc + b * g.R * g.sc_bytes, &maps[i].scale, kb / 32, row0, bar);
        tma_load_2d(dst + g.off_mn + b * g.R * g.sc_bytes, &maps[i].mn, kb / 32, row0, bar);
      }
    }
  }
}

// Adds one stage's share of warp (row r, part p of WPR) to acc[NM][MT]: its
// chunks of the stage (chunk = 32 INT4 or 16 INT8 codes, one per lane per
// pass) times the staged activations of the stage's K range (chunk index
// c0 + chunk within the staged row).
template <int FMT, int MT, int NM>
__device__ __forceinline__ void stage_dot(const Geo& g, const uint8_t* st, int r, int p, int wpr, int lane,
                                          const uint8_t* xi, int tok_stride, const float* xf, const float* xsum,
                                          int nch_row, int c0, float (&acc)[2][2]) {
  using C = Codes<FMT>;
  const int nch = g.kc / C::kChunk;        // chunks of a row in the stage
  const int per = nch / wpr;               // chunks of this warp
  const int cpb = g.box / C::kChunk;       // chunks per box
  for (int cl = lane; cl < per; cl += 32) {
    const int ch = p * per + cl;
    const int bx = ch / cpb, cb = ch - bx * cpb;
    const int c = c0 + ch;                 // chunk index within the staged activation row
#pragma unroll
    for (int i = 0; i < NM; ++i) {
      const int b = i * g.nbox + bx;
      const uint4 wv = *reinterpret_cast<const uint4*>(st + (b * g.R + r) * g.code_bytes + cb * 16);
      float sc = 1.f, mn = 0.f;
      if (FMT == FMT_INT4_G32) {
        sc = __half2float(*reinterpret_cast<const __half*>(st + g.off_sc + (b * g.R + r) * g.sc_bytes + cb * 2));
        mn = __half2float(*reinterpret_cast<const __half*>(st + g.off_mn + (b * g.R + r) * g.sc_bytes + cb * 2));
      }
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const float P = (float)chunk_dot<FMT>(wv, xi + t * tok_stride + c * C::kStageBytes);   // exact below 2^24
        const float f = xf[t * nch_row + c];
        // sum_k (q_k s + m) x_k = s * 2^(e-14) * sum_k q_k xi_k + m * sum_k x_k
        acc[i][t] = FMT == FMT_INT4_G32 ? fmaf(sc * f, P, fmaf(mn, xsum[t * nch_row + c], acc[i][t]))
                                        : fmaf(f, P, acc[i][t]);
      }
    }
  }
}

template <int FMT, int MT, int MODE>
__global__ void __launch_bounds__(kThreads, 1) k_ffn_stream(const __grid_constant__ FfnStreamArgs a) {
  using C = Codes<FMT>;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int S = a.stages;

  const Geo ga = make_geo<FMT>(kRowsA, 2, a.kc_a, a.box_a);
  const Geo gb = make_geo<FMT>(kRowsB, 1, a.kc_b, a.box_b);
  const int a_lo = (int)((long long)blockIdx.x * a.blocks_a / G), a_hi = (int)((long long)(blockIdx.x + 1) * a.blocks_a / G);
  const int b_lo = (int)((long long)blockIdx.x * a.blocks_b / G), b_hi = (int)((long long)(blockIdx.x + 1) * a.blocks_b / G);
  const int nja = a.H / a.kc_a, njb = a.I / a.kc_b;   // stages per row block
  const int stages_a = (a_hi - a_lo) * nja, stages_b = (b_hi - b_lo) * njb;

  // ---- shared memory carve ------------------------------------------------
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + 8;
  float* red = reinterpret_cast<float*>(smem + 128);              // [2][16 warps][2][MT]
  uint8_t* xs = smem + 128 + 2 * kConsumerWarps * 2 * MT * 4 + 128;
  xs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(xs) + 127) & ~uintptr_t(127));
  uint8_t* ring = xs + a.stage_x_bytes;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      const int total = stages_a + stages_b;
      for (int s = 0; s < total; ++s) {
        const int slot = s % S, use = s / S;
        if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1)) break;
        uint8_t* dst = ring + (size_t)slot * a.stage_bytes;
        if (s < stages_a) {
          const int b = a_lo + s / nja, j = s % nja;
          load_stage<FMT>(ga, a.maps_a, dst, b * kRowsA, j * a.kc_a, &full[slot]);
        } else {
          const int sb = s - stages_a;
          const int b = b_lo + sb / njb, j = sb % njb;
          load_stage<FMT>(gb, &a.map_down, dst, b * kRowsB, j * a.kc_b, &full[slot]);
        }
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ct = threadIdx.x;                       // 0..511
  constexpr int kCT = 32 * kConsumerWarps;
  const int ncha = a.H / C::kChunk, nchb = a.I / C::kChunk;
  bool dead = false;

  // Stage x (all H) for phase A.
  {
    const int tok_stride = ncha * C::kStageBytes;
    float* xf = reinterpret_cast<float*>(xs + MT * tok_stride);
    float* xsum = xf + MT * ncha;
    for (int i = ct; i < MT * ncha; i += kCT) {
      const int t = i / ncha, c = i - t * ncha;
      stage_chunk<FMT>(a.x + (size_t)t * a.H + c * C::kChunk, xs + t * tok_stride + c * C::kStageBytes, &xf[i],
                       &xsum[i]);
    }
  }
  named_sync(1, kCT);

  int s = 0;   // stage counter (ring position)
  // ---- phase A: gate/up rows, h = act(g, u) ----
  {
    const int tok_stride = ncha * C::kStageBytes;
    const float* xf = reinterpret_cast<const float*>(xs + MT * tok_stride);
    const float* xsum = xf + MT * ncha;
    const int r = warp / kWarpsPerRowA, p = warp % kWarpsPerRowA;
    int blk = 0;
    for (int b = a_lo; b < a_hi; ++b, ++blk) {
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      for (int j = 0; j < nja; ++j, ++s) {
        const int slot = s % S, use = s / S;
        if (!dead && !mbar_wait(&full[slot], use & 1)) dead = true;
        if (!dead)
          stage_dot<FMT, MT, 2>(ga, ring + (size_t)slot * a.stage_bytes, r, p, kWarpsPerRowA, lane, xs, tok_stride, xf,
                                xsum, ncha, j * (a.kc_a / C::kChunk), acc);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      // The row's warps meet on their own barrier (ids 2..9); the first of
      // them combines the parts.
      float* rb = red + (blk & 1) * (kConsumerWarps * 2 * MT);
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const float v = warp_sum(acc[i][t]);
          if (lane == 0) rb[(warp * 2 + i) * MT + t] = v;
        }
      named_sync(2 + r, 32 * kWarpsPerRowA);
      if (p == 0 && lane < MT) {
        const int rr = r, t = lane;
        const int row = b * kRowsA + rr;
        if (row < a.I) {
          float g = 0.f, u = 0.f;
          for (int q = 0; q < kWarpsPerRowA; ++q) {
            g += rb[((rr * kWarpsPerRowA + q) * 2 + 0) * MT + t];
            u += rb[((rr * kWarpsPerRowA + q) * 2 + 1) * MT + t];
          }
          if (FMT == FMT_INT8_ROW) {
            g *= __half2float(a.rs_gate[row]);
            u *= __half2float(a.rs_up[row]);
          }
          a.hbuf[(size_t)t * a.I + row] = float_to_bf16_bits(gated_act(g, u, a.act));
        }
      }
    }
  }

  // ---- all of h written: stage it for phase B ----
  if (!grid_barrier(0, ct)) dead = true;
  {
    const int tok_stride = nchb * C::kStageBytes;
    float* xf = reinterpret_cast<float*>(xs + MT * tok_stride);
    float* xsum = xf + MT * nchb;
    for (int i = ct; i < MT * nchb; i += kCT) {
      const int t = i / nchb, c = i - t * nchb;
      stage_chunk<FMT>(a.hbuf + (size_t)t * a.I + c * C::kChunk, xs + t * tok_stride + c * C::kStageBytes, &xf[i],
                       &xsum[i]);
    }
  }
  named_sync(1, kCT);

  // ---- phase B: down rows ----
  {
    const int tok_stride = nchb * C::kStageBytes;
    const float* xf = reinterpret_cast<const float*>(xs + MT * tok_stride);
    const float* xsum = xf + MT * nchb;
    const int r = warp / kWarpsPerRowB, p = warp % kWarpsPerRowB;
    int blk = 0;
    for (int b = b_lo; b < b_hi; ++b, ++blk) {
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
      for (int j = 0; j < njb; ++j, ++s) {
        const int slot = s % S, use = s / S;
        if (!dead && !mbar_wait(&full[slot], use & 1)) dead = true;
        if (!dead)
          stage_dot<FMT, MT, 1>(gb, ring + (size_t)slot * a.stage_bytes, r, p, kWarpsPerRowB, lane, xs, tok_stride, xf,
                                xsum, nchb, j * (a.kc_b / C::kChunk), acc);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      float* rb = red + (blk & 1) * (kConsumerWarps * 2 * MT);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const float v = warp_sum(acc[0][t]);
        if (lane == 0) rb[(warp * 2) * MT + t] = v;
      }
      named_sync(2 + r, 32 * kWarpsPerRowB);
      if (p == 0 && lane < MT) {
        const int rr = r, t = lane;
        const int row = b * kRowsB + rr;
        if (row < a.H) {
          float y = 0.f;
          for (int q = 0; q < kWarpsPerRowB; ++q) y += rb[((rr * kWarpsPerRowB + q) * 2) * MT + t];
          if (FMT == FMT_INT8_ROW) y *= __half2float(a.rs_down[row]);
          const float yb = round_bf16(y);
          const size_t o = (size_t)t * a.H + row;
          if (MODE == STREAM_RESIDUAL) {
            a.res[o] = float_to_bf16_bits(bf16_bits_to_float(a.res[o]) + yb);
          } else {
            a.ybuf[o] = yb;
          }
        }
      }
    }
  }

  if (MODE == STREAM_RMSNORM) {
    // out = bf16(y / sqrt(mean(y^2) + eps) * w) over the whole row of H.
    if (!grid_barrier(1, ct)) dead = true;
    float* red2 = red;   // [16 warps][MT]
    float ss[2] = {0.f, 0.f};
    for (int n = ct; n < a.H; n += kCT)
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const float y = __ldcg(a.ybuf + (size_t)t * a.H + n);
        ss[t] = fmaf(y, y, ss[t]);
      }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const float v = warp_sum(ss[t]);
      if (lane == 0) red2[warp * MT + t] = v;
    }
    named_sync(1, kCT);
    for (int i = ct; i < MT * (b_hi - b_lo) * kRowsB; i += kCT) {
      const int t = i % MT, row = b_lo * kRowsB + i / MT;
      if (row >= a.H) continue;
      float tot = 0.f;
      for (int w = 0; w < kConsumerWarps; ++w) tot += red2[w * MT + t];
      const float inv_rms = 1.0f / sqrtf(tot / (float)a.H + a.eps);
      const size_t o = (size_t)t * a.H + row;
      a.out[o] = float_to_bf16_bits(__ldcg(a.ybuf + o) * inv_rms * bf16_bits_to_float(a.norm_w[row]));
    }
  }
}

template <int FMT, int MT, int MODE>
cudaError_t launch_t(const FfnStreamArgs& a, int grid, size_t smem, cudaStream_t s) {
  auto kern = k_ffn_stream<FMT, MT, MODE>;
  // Opt in to what this launch needs (the kernel also has a little static
  // shared memory, which counts against the same per-block limit).
  static size_t smem_set = 0;
  if (smem > smem_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    smem_set = smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

template <int FMT, int MODE>
cudaError_t launch_mt(const FfnStreamArgs& a, int grid, size_t smem, cudaStream_t s) {
  return a.M == 2 ? launch_t<FMT, 2, MODE>(a, grid, smem, s) : launch_t<FMT, 1, MODE>(a, grid, smem, s);
}

// Largest divisor of n that is at most cap and a multiple of step (0: none).
int divisor_at_most(int n, int cap, int step) {
  for (int d = cap / step * step; d >= step; d -= step)
    if (n % d == 0) return d;
  return 0;
}

constexpr int kRingBytes = 160 * 1024;   // weight bytes in flight per SM
constexpr size_t kSmemMax = 227 * 1024 - 1024;   // room for the static shared memory

}  // namespace

bool ffn_stream_plan(FfnStreamArgs* a, int fmt, int H, int I, int M) {
  if (M < 1 || M > 2) return false;
  const bool i4 = fmt == FMT_INT4_G32;
  if (!i4 && fmt != FMT_INT8_ROW) return false;
  const int chunk = i4 ? 32 : 16;
  const int box_max = i4 ? 4096 : 2048;        // 256 eight-byte elements per box row
  // Phase A: 8 row pairs x kc_a; two warps per row, whole chunks per warp.
  const int kc_a = divisor_at_most(H, i4 ? 2048 : 1024, i4 ? 256 : kWarpsPerRowA * chunk);
  // Phase B: 4 rows x kc_b; four warps per row.
  const int kc_b = divisor_at_most(I, i4 ? 7168 : 4096, i4 ? 256 : kWarpsPerRowB * chunk);
  if (kc_a == 0 || kc_b == 0) return false;
  if ((kc_a / chunk) % kWarpsPerRowA != 0 || (kc_b / chunk) % kWarpsPerRowB != 0) return false;
  const int box_a = divisor_at_most(kc_a, box_max, i4 ? 256 : 8);
  const int box_b = divisor_at_most(kc_b, box_max, i4 ? 256 : 8);
  if (box_a == 0 || box_b == 0 || box_a % chunk != 0 || box_b % chunk != 0) return false;
  // Every TMA box of a stage lands on a 128-byte boundary.
  auto aligned = [&](int R, int NM, int kc, int box) {
    const int code_bytes = i4 ? box / 2 : box, sc_bytes = i4 ? box / 16 : 0, boxes = NM * (kc / box);
    return (R * code_bytes) % 128 == 0 && (R * sc_bytes) % 128 == 0 && (boxes * R * code_bytes) % 128 == 0;
  };
  if (!aligned(kRowsA, 2, kc_a, box_a) || !aligned(kRowsB, 1, kc_b, box_b)) return false;
  const double bpc = i4 ? 0.625 : 1.0;          // stage bytes per code (codes + scales + mins)
  const int bytes_a = (int)(2 * kRowsA * kc_a * bpc), bytes_b = (int)(kRowsB * kc_b * bpc);
  const int stage_bytes = (std::max(bytes_a, bytes_b) + 127) / 128 * 128;
  const int cbytes = i4 ? 80 : 48;
  auto stage_x = [&](int K) {
    const int nch = K / chunk;
    return ((size_t)M * nch * cbytes + (size_t)M * nch * 4 * (i4 ? 2 : 1) + 127) / 128 * 128;
  };
  const size_t sx = std::max(stage_x(H), stage_x(I));
  const size_t fixed = 128 + 2 * 16 * 2 * 2 * 4 + 256 + sx;
  int stages = std::min(8, kRingBytes / stage_bytes);
  while (stages > 2 && fixed + (size_t)stages * stage_bytes > kSmemMax) --stages;
  if (stages < 2 || fixed + (size_t)stages * stage_bytes > kSmemMax) return false;
  a->H = H; a->I = I; a->M = M;
  a->kc_a = kc_a; a->box_a = box_a; a->kc_b = kc_b; a->box_b = box_b;
  a->blocks_a = (I + kRowsA - 1) / kRowsA;
  a->blocks_b = (H + kRowsB - 1) / kRowsB;
  a->stage_bytes = stage_bytes;
  a->stage_x_bytes = (int)sx;
  a->stages = stages;
  a->smem = fixed + (size_t)stages * stage_bytes;
  return true;
}

cudaError_t ffn_stream_encode(FfnStreamArgs* a, int fmt, const QW& gate, const QW& up, const QW& down) {
  auto enc = [&](QWMaps* m, const QW& w, int N, int K, int box, int rows) -> cudaError_t {
    cudaError_t e;
    if (fmt == FMT_INT4_G32) {
      e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT64, w.q, K / 16, N, K / 2, box / 16, rows);
      if (e != cudaSuccess) return e;
      e = encode_tmap_2d(&m->scale, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.scale, K / 32, N, K / 16, box / 32, rows);
      if (e != cudaSuccess) return e;
      return encode_tmap_2d(&m->mn, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.mn, K / 32, N, K / 16, box / 32, rows);
    }
    e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT64, w.q, K / 8, N, K, box / 8, rows);
    m->scale = m->codes;
    m->mn = m->codes;
    return e;
  };
  cudaError_t e = enc(&a->maps_a[0], gate, a->I, a->H, a->box_a, kRowsA);
  if (e == cudaSuccess) e = enc(&a->maps_a[1], up, a->I, a->H, a->box_a, kRowsA);
  if (e == cudaSuccess) e = enc(&a->map_down, down, a->H, a->I, a->box_b, kRowsB);
  return e;
}

cudaError_t launch_ffn_stream(const FfnStreamArgs& a, int fmt, int mode, cudaStream_t s) {
  static int sms[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (sms[dev] == 0) {
    e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  if (fmt == FMT_INT4_G32)
    return mode == STREAM_RMSNORM ? launch_mt<FMT_INT4_G32, STREAM_RMSNORM>(a, sms[dev], a.smem, s)
                                  : launch_mt<FMT_INT4_G32, STREAM_RESIDUAL>(a, sms[dev], a.smem, s);
  return mode == STREAM_RMSNORM ? launch_mt<FMT_INT8_ROW, STREAM_RMSNORM>(a, sms[dev], a.smem, s)
                                : launch_mt<FMT_INT8_ROW, STREAM_RESIDUAL>(a, sms[dev], a.smem, s);
}

unsigned int ffn_stream_fault_flags(bool clear) {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_fault_flags, sizeof(v));
  if (clear && v) {
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_fault_flags, &z, sizeof(z));
    // A barrier that timed out may have left an arrival count behind.
    const unsigned long long zero[4] = {0, 0, 0, 0};
    cudaMemcpyToSymbol(g_grid_bar, zero, sizeof(zero));
  }
  return v;
}

}  // namespace moeffn
