// Quantized GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), for
// several token rows per weight matrix (prefill, batched decode, and the
// grouped expert GEMMs of the MoE layer).
//
// Operand roles: the MMA's M dimension (128) runs over token rows (A, bf16
// activations loaded by TMA) and its N dimension over weight rows (B, up to
// 256 dequantized rows per tile). A tcgen05.mma occupies the tensor core for
// about the same time whatever its N up to 256, so putting the weights on N
// halves the instruction count per weight against weights on M.
// Per CTA: one tile of weight rows x MT tiles of 128 token rows x the job's K
// range (or one K split of it).
//
//  warp 0      weight producer: TMA loads of the quantized weight stages
//              (codes in 128-byte swizzled boxes, INT4 group scales and mins);
//  warp 2      token producer: TMA loads of the bf16 token tiles (128-byte
//              swizzled, the MMA's A operand);
//  warp 1      allocates the TMEM accumulators and issues tcgen05.mma (one
//              thread), releasing operand slots with tcgen05.commit;
//  warps 4-19  dequantize: two threads per weight row each write 32 bf16
//              weights of the K atom (w = RNE(q * scale + min), exact in fp32
//              before the rounding) into the swizzled canonical layout the MMA
//              reads; then, as the epilogue, read TMEM (warp w sees lanes
//              32*(w%4)..+31, one quarter of the token rows) and write the
//              outputs, the four warps of a lane quarter sharing the columns.
//
// Modes: GATEUP stacks F gate rows and the same F up rows in one 2F-row B
// tile, so a token's gate and up sums sit in one TMEM lane (columns j and
// F + j) and the epilogue writes bf16(act(gate) * up). DOWN writes fp32
// partial sums d[split][slot][row] that the layer tails combine. INT8-row
// weights enter the MMA as their exact integer codes and are scaled per
// column in the epilogue.
#include "gemm_tc.cuh"
#include "launch.cuh"
#include "sync.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace moeffn {

namespace {

constexpr int kDqWarps = 16;                  // warps 4..19
constexpr int kThreads = 32 * (4 + kDqWarps);
constexpr int kTokRows = 128;                 // MMA M: token rows per tile
constexpr int kMaxRows = 256;                 // MMA N: weight rows per tile
constexpr int kBAtomBytes = kMaxRows * 128;   // one K atom (64) of dequantized weights
constexpr int kAAtomBytes = kTokRows * 128;   // one K atom of one token tile

template <int FMT>
struct TcFmt;
template <>
struct TcFmt<FMT_INT4_G32> {
  static constexpr int kKTile = 256;      // codes per weight stage row (128 bytes)
  static constexpr int kAtoms = 4;        // K atoms of 64 per stage
  static constexpr int kCodeBytes = kMaxRows * 128;
  static constexpr int kScaleBytes = kMaxRows * 16;
  static constexpr int kStageBytes = kCodeBytes + 2 * kScaleBytes;
  static constexpr int kRowBytes = 128 + 2 * 16;   // bytes a stage loads per weight row
};
template <>
struct TcFmt<FMT_INT8_ROW> {
  static constexpr int kKTile = 128;
  static constexpr int kAtoms = 2;
  static constexpr int kCodeBytes = kMaxRows * 128;
  static constexpr int kScaleBytes = 0;
  static constexpr int kStageBytes = kCodeBytes;
  static constexpr int kRowBytes = 128;
};

template <int MT>
struct TcPipe {
  static constexpr int kSW = 2;                  // quantized weight stages
  static constexpr int kSB = MT == 1 ? 3 : 2;    // dequantized weight atoms
  static constexpr int kSA = MT == 1 ? 3 : 2;    // token atoms (MT tiles each)
  static constexpr uint32_t kTmemCols = 256u * MT;
};

template <int FMT, int MT>
constexpr size_t tc_smem_bytes() {
  return 1024 /*align slack*/ + 1024 /*barriers*/ + (size_t)TcPipe<MT>::kSW * TcFmt<FMT>::kStageBytes +
         (size_t)TcPipe<MT>::kSB * kBAtomBytes + (size_t)TcPipe<MT>::kSA * MT * kAAtomBytes;
}
static_assert(tc_smem_bytes<FMT_INT4_G32, 1>() <= 232448, "shared memory");
static_assert(tc_smem_bytes<FMT_INT4_G32, 2>() <= 232448, "shared memory");
static_assert(tc_smem_bytes<FMT_INT8_ROW, 1>() <= 232448, "shared memory");
static_assert(tc_smem_bytes<FMT_INT8_ROW, 2>() <= 232448, "shared memory");

struct Job {
  const TcMaps* m0;
  const TcMaps* m1;
  const CUtensorMap* xmap;
  const __half* rs0;
  const __half* rs1;
  int N, K, ntok, slot0, tile;
  bool shared, valid;
};

__device__ __forceinline__ Job decode_job(const TcGemmArgs& a) {
  Job j{};
  j.valid = true;
  const int z = blockIdx.z;
  if (a.offsets == nullptr) {
    j.m0 = &a.w0; j.m1 = &a.w1; j.xmap = &a.xmap; j.rs0 = a.rscale0; j.rs1 = a.rscale1;
    j.N = a.N; j.K = a.K; j.ntok = a.M; j.tile = a.tile;
  } else if (z < a.routed_jobs) {
    if (z >= *a.n_union) { j.valid = false; return j; }
    const int e = a.union_list[z];
    j.m0 = a.tab0 + e;
    j.m1 = a.tab1 != nullptr ? a.tab1 + e : nullptr;
    j.xmap = &a.xmap;
    j.N = a.N; j.K = a.K; j.tile = a.tile;
    j.slot0 = a.offsets[e];
    j.ntok = a.offsets[e + 1] - j.slot0;
  } else {
    j.m0 = &a.s0; j.m1 = &a.s1; j.xmap = &a.xmap_s;
    j.N = a.Ns; j.K = a.Ks; j.ntok = a.M; j.tile = a.tile_s; j.shared = true;
  }
  return j;
}

// ---- dequantization of one K atom (64 weights) of one row into the B tile ----

// INT4: half hf of atom j is group g = 2j + hf of the stage row (one 16-byte
// chunk of the 128-byte swizzled row, 32 codes); w = q * s + m in fp32
// (exact), rounded to bf16, written as chunks 4hf..4hf+3 of the atom row.
__device__ __forceinline__ void dequant_half_int4(uint32_t wq, int r, int j, int hf, uint32_t b_atom) {
  const uint32_t code_row = wq + r * 128;
  const int g = 2 * j + hf;
  const uint32_t sw = lds_u32(wq + TcFmt<FMT_INT4_G32>::kCodeBytes + r * 16 + (g >> 1) * 4);
  const uint32_t mw =
      lds_u32(wq + TcFmt<FMT_INT4_G32>::kCodeBytes + TcFmt<FMT_INT4_G32>::kScaleBytes + r * 16 + (g >> 1) * 4);
  const float s = __half2float(__ushort_as_half((unsigned short)((sw >> ((g & 1) * 16)) & 0xFFFFu)));
  const float m = __half2float(__ushort_as_half((unsigned short)((mw >> ((g & 1) * 16)) & 0xFFFFu)));
  const uint4 cw = lds_u128(code_row + (((g ^ (r & 7)) & 7) << 4));
  const uint32_t brow = b_atom + r * 128;
  const uint32_t mg = kMagic, m0 = 0x000Fu, m1 = 0x00F0u, m2 = 0x0F00u, m3 = 0xF000u;
  // The magic conversion leaves code i of a half-word scaled by 16^(i%4):
  // undo it in the scale (exact powers of two).
  const float2 s01 = make_float2(s, s * 0.0625f), s23 = make_float2(s * 0.00390625f, s * 0.000244140625f);
  const float2 mm = make_float2(m, m), sub = make_float2(-kMagicF, -kMagicF);
  const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t w = words[q], hi = w >> 16;
    float2 c01 = make_float2(__uint_as_float(and_or(w, m0, mg)), __uint_as_float(and_or(w, m1, mg)));
    float2 c23 = make_float2(__uint_as_float(and_or(w, m2, mg)), __uint_as_float(and_or(w, m3, mg)));
    float2 c45 = make_float2(__uint_as_float(and_or(hi, m0, mg)), __uint_as_float(and_or(hi, m1, mg)));
    float2 c67 = make_float2(__uint_as_float(and_or(hi, m2, mg)), __uint_as_float(and_or(hi, m3, mg)));
    c01 = __ffma2_rn(__fadd2_rn(c01, sub), s01, mm);
    c23 = __ffma2_rn(__fadd2_rn(c23, sub), s23, mm);
    c45 = __ffma2_rn(__fadd2_rn(c45, sub), s01, mm);
    c67 = __ffma2_rn(__fadd2_rn(c67, sub), s23, mm);
    const uint4 out = make_uint4(pack_bf16x2(c01.x, c01.y), pack_bf16x2(c23.x, c23.y), pack_bf16x2(c45.x, c45.y),
                                 pack_bf16x2(c67.x, c67.y));
    const int chunk = 4 * hf + q;  // 8 bf16 = 16 bytes of the 128-byte atom row
    sts_u128(brow + ((chunk ^ (r & 7)) << 4), out);
  }
}

// INT8: half hf of atom j is input chunks 4j+2hf, 4j+2hf+1 (32 signed codes)
// as exact bf16 integers; the row scale is applied in the epilogue.
__device__ __forceinline__ void dequant_half_int8(uint32_t wq, int r, int j, int hf, uint32_t b_atom) {
  const uint32_t code_row = wq + r * 128;
  const uint32_t brow = b_atom + r * 128;
  const uint32_t mg = kMagic;
  const float2 sub = make_float2(-(kMagicF + 128.0f), -(kMagicF + 128.0f));
#pragma unroll
  for (int cc = 0; cc < 2; ++cc) {
    const int c = 2 * hf + cc;                 // 16-code chunk within the atom
    const int chunk_in = 4 * j + c;
    const uint4 cw = lds_u128(code_row + (((chunk_in ^ (r & 7)) & 7) << 4));
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    uint32_t packed[8];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t u = words[q] ^ 0x80808080u;  // byte = q + 128
      uint32_t b0, b1, b2, b3;
      asm("prmt.b32 %0, %1, %2, 0x7540;" : "=r"(b0) : "r"(u), "r"(mg));
      asm("prmt.b32 %0, %1, %2, 0x7541;" : "=r"(b1) : "r"(u), "r"(mg));
      asm("prmt.b32 %0, %1, %2, 0x7542;" : "=r"(b2) : "r"(u), "r"(mg));
      asm("prmt.b32 %0, %1, %2, 0x7543;" : "=r"(b3) : "r"(u), "r"(mg));
      const float2 v01 = __fadd2_rn(make_float2(__uint_as_float(b0), __uint_as_float(b1)), sub);
      const float2 v23 = __fadd2_rn(make_float2(__uint_as_float(b2), __uint_as_float(b3)), sub);
      packed[2 * q] = pack_bf16x2(v01.x, v01.y);
      packed[2 * q + 1] = pack_bf16x2(v23.x, v23.y);
    }
    const int ch0 = 2 * c, ch1 = 2 * c + 1;  // 16 codes -> two 16-byte chunks of the atom row
    sts_u128(brow + ((ch0 ^ (r & 7)) << 4), make_uint4(packed[0], packed[1], packed[2], packed[3]));
    sts_u128(brow + ((ch1 ^ (r & 7)) << 4), make_uint4(packed[4], packed[5], packed[6], packed[7]));
  }
}

// Eight consecutive fp16 scales from global memory (16-byte aligned).
__device__ __forceinline__ void load_scales8(const __half* p, float (&s)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s[2 * i] = __half2float(__ushort_as_half((unsigned short)(w[i] & 0xFFFFu)));
    s[2 * i + 1] = __half2float(__ushort_as_half((unsigned short)(w[i] >> 16)));
  }
}

template <int FMT, int MT, int MODE>
__global__ void __launch_bounds__(kThreads, 1) k_qgemm_tc(const __grid_constant__ TcGemmArgs a) {
  using F = TcFmt<FMT>;
  using P = TcPipe<MT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  pdl_wait();
  const Job job = decode_job(a);
  if (!job.valid) return;
  const int tt = blockIdx.y % a.token_tiles, split = blockIdx.y / a.token_tiles;
  const int t0 = tt * (MT * kTokRows);
  if (t0 >= job.ntok) return;
  // Weight rows of the tile: F gate + F up features (GATEUP) or R outputs.
  const int feat = job.tile;
  const int nrows = (MODE == TC_GATEUP) ? 2 * feat : feat;
  const int n0 = blockIdx.x * feat;
  if (n0 >= job.N) return;
  const int k0 = split * a.ks_len;
  if (k0 >= job.K) return;
  const int klen = min(a.ks_len, job.K - k0);
  const int nk = klen / 64;                                  // K atoms (klen is a multiple of the stage K)
  const int tn = min(MT * kTokRows, job.ntok - t0);          // valid token rows
  const int mt = (tn + kTokRows - 1) / kTokRows;             // token tiles holding rows (1..MT)

  // ---- shared memory carve (1024-byte aligned operand tiles) -------------
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_addr(smem_raw));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase);
  uint64_t* wq_full = bars;
  uint64_t* wq_empty = wq_full + P::kSW;
  uint64_t* b_full = wq_empty + P::kSW;
  uint64_t* b_empty = b_full + P::kSB;
  uint64_t* a_full = b_empty + P::kSB;
  uint64_t* a_empty = a_full + P::kSA;
  uint64_t* acc_full = a_empty + P::kSA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + 512);
  const uint32_t wq_base = base + 1024;
  const uint32_t b_base = wq_base + P::kSW * F::kStageBytes;
  const uint32_t a_base = b_base + P::kSB * kBAtomBytes;
  constexpr uint32_t kASlotBytes = MT * kAAtomBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < P::kSW; ++i) { mbar_init(&wq_full[i], 1); mbar_init(&wq_empty[i], kDqWarps); }
    for (int i = 0; i < P::kSB; ++i) { mbar_init(&b_full[i], kDqWarps); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < P::kSA; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, P::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  const int row_tok = job.slot0 + t0;   // first token row (token or slot) of the tile

  if (warp == 0) {
    // ---------------- weight producer ----------------
    if (lane == 0) {
      const int nw = nk / F::kAtoms;
      const uint32_t tx = (uint32_t)nrows * F::kRowBytes;
      for (int w = 0; w < nw; ++w) {
        const int slot = w % P::kSW, use = w / P::kSW;
        if (use > 0 && !mbar_wait_spin(&wq_empty[slot], (use - 1) & 1)) break;
        uint8_t* gst = gbase + (wq_base - base) + slot * F::kStageBytes;
        mbar_arrive_expect_tx(&wq_full[slot], tx);
        const int kc = k0 + w * F::kKTile;                 // first K element of the stage
        const int cx = (FMT == FMT_INT4_G32) ? kc / 2 : kc; // byte column of the codes
        tma_load_2d(gst, &job.m0->codes, cx, n0, &wq_full[slot]);
        if (MODE == TC_GATEUP) tma_load_2d(gst + feat * 128, &job.m1->codes, cx, n0, &wq_full[slot]);
        if (FMT == FMT_INT4_G32) {
          uint8_t* gs = gst + F::kCodeBytes;
          tma_load_2d(gs, &job.m0->scale, kc / 32, n0, &wq_full[slot]);
          tma_load_2d(gs + F::kScaleBytes, &job.m0->mn, kc / 32, n0, &wq_full[slot]);
          if (MODE == TC_GATEUP) {
            tma_load_2d(gs + feat * 16, &job.m1->scale, kc / 32, n0, &wq_full[slot]);
            tma_load_2d(gs + F::kScaleBytes + feat * 16, &job.m1->mn, kc / 32, n0, &wq_full[slot]);
          }
        }
      }
    }
  } else if (warp == 2) {
    // ---------------- token producer ----------------
    if (lane == 0) {
      for (int k = 0; k < nk; ++k) {
        const int slot = k % P::kSA, use = k / P::kSA;
        if (use > 0 && !mbar_wait_spin(&a_empty[slot], (use - 1) & 1)) break;
        mbar_arrive_expect_tx(&a_full[slot], (uint32_t)mt * kAAtomBytes);
        uint8_t* dst = gbase + (a_base - base) + slot * kASlotBytes;
        for (int t = 0; t < mt; ++t)
          tma_load_2d(dst + t * kAAtomBytes, job.xmap, k0 + k * 64, row_tok + t * kTokRows, &a_full[slot]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    // The barrier polls for atom k+1 are made while atom k's MMAs run (before
    // its last MMA is issued) instead of after them.
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kTokRows, nrows);
      bool ok = mbar_wait_spin(&b_full[0], 0) && mbar_wait_spin(&a_full[0], 0);
      for (int k = 0; k < nk && ok; ++k) {
        const int bs = k % P::kSB, as = k % P::kSA;
        tc_fence_after();
        const uint64_t bd = umma_desc_sw128(b_base + bs * kBAtomBytes);
        const uint64_t ad = umma_desc_sw128(a_base + as * kASlotBytes);
        const uint32_t acc0 = k != 0;
        for (int t = 0; t < mt; ++t) {
          const uint64_t adt = ad + (uint64_t)((t * kAAtomBytes) >> 4);
          const uint32_t dt = tmem + (uint32_t)(t * kMaxRows);
#pragma unroll
          for (int kk = 0; kk < 3; ++kk)   // K=16 steps of 32 bytes inside the 128-byte swizzled row
            umma_bf16(dt, adt + 2 * kk, bd + 2 * kk, idesc, acc0 | (kk != 0 ? 1u : 0u));
          if (t + 1 < mt) umma_bf16(dt, adt + 6, bd + 6, idesc, 1u);
        }
        const int kn = k + 1;
        const bool next_ok = kn >= nk || (mbar_wait_spin(&b_full[kn % P::kSB], (kn / P::kSB) & 1) &&
                                          mbar_wait_spin(&a_full[kn % P::kSA], (kn / P::kSA) & 1));
        umma_bf16(tmem + (uint32_t)((mt - 1) * kMaxRows), ad + (uint64_t)(((mt - 1) * kAAtomBytes) >> 4) + 6, bd + 6,
                  idesc, 1u);
        umma_commit(&b_empty[bs]);
        umma_commit(&a_empty[as]);
        if (!next_ok) ok = false;
        else if (kn == nk) umma_commit(acc_full);
      }
    }
  } else if (warp >= 4) {
    // ---------------- dequantize (warps 4-19), then epilogue ----------------
    const int d = threadIdx.x - 128;
    const int r = d & (kMaxRows - 1), hf = d >> 8;   // weight row of the B tile, half of the atom row
    const bool active = r < nrows;
    bool dead = false;
    for (int k = 0; k < nk; ++k) {
      const int w = k / F::kAtoms, j = k % F::kAtoms, ws = w % P::kSW;
      const int bs = k % P::kSB, buse = k / P::kSB;
      if (!dead && j == 0 && !mbar_wait_spin(&wq_full[ws], (w / P::kSW) & 1)) dead = true;
      if (!dead && buse > 0 && !mbar_wait_spin(&b_empty[bs], (buse - 1) & 1)) dead = true;
      if (!dead && active) {
        const uint32_t wq = wq_base + ws * F::kStageBytes;
        if (FMT == FMT_INT4_G32) dequant_half_int4(wq, r, j, hf, b_base + bs * kBAtomBytes);
        else dequant_half_int8(wq, r, j, hf, b_base + bs * kBAtomBytes);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&b_full[bs]);
        if (j == F::kAtoms - 1) mbar_arrive(&wq_empty[ws]);
      }
    }
    // Epilogue: TMEM lanes = token rows, columns = weight rows of the tile.
    if (!dead && !mbar_wait(acc_full, 0)) dead = true;
    dead = __any_sync(0xffffffffu, dead);   // TMEM loads are warp-collective
    tc_fence_after();
    const int q4 = warp & 3, share = (warp - 4) >> 2;   // lane quarter, column share
    const int nchunks = feat / 8;                       // 8-column chunks of outputs
    for (int t = 0; t < mt && !dead; ++t) {
      const int tok = t * kTokRows + 32 * q4 + lane;    // token row within the CTA's range
      const bool valid = tok < tn;
      const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16) + (uint32_t)(t * kMaxRows);
      for (int c = share; c < nchunks; c += 4) {
        const int n = n0 + 8 * c;
        float v[8];
        tmem_ld8(trow + 8 * c, v);
        if (MODE == TC_GATEUP) {
          float u[8];
          tmem_ld8(trow + feat + 8 * c, u);
          if (valid && n < job.N) {
            if (FMT == FMT_INT8_ROW) {
              float sg[8], su[8];
              load_scales8(job.rs0 + n, sg);
              load_scales8(job.rs1 + n, su);
#pragma unroll
              for (int i = 0; i < 8; ++i) { v[i] *= sg[i]; u[i] *= su[i]; }
            }
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
              o[i] = (uint32_t)float_to_bf16_bits(gated_act(v[2 * i], u[2 * i], a.act)) |
                     ((uint32_t)float_to_bf16_bits(gated_act(v[2 * i + 1], u[2 * i + 1], a.act)) << 16);
            uint16_t* out = job.shared ? a.out_act_s : a.out_act;
            *reinterpret_cast<uint4*>(out + (size_t)(row_tok + tok) * job.N + n) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        } else if (valid && n < job.N) {
          if (FMT == FMT_INT8_ROW) {
            float sd[8];
            load_scales8(job.rs0 + n, sd);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] *= sd[i];
          }
          float* dout = job.shared ? a.out_d_s : a.out_d;
          const int nslots = job.shared ? a.M : a.slots;
          float4* p = reinterpret_cast<float4*>(dout + ((size_t)split * nslots + row_tok + tok) * job.N + n);
          p[0] = make_float4(v[0], v[1], v[2], v[3]);
          p[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, P::kTmemCols);
  }
}

template <int FMT, int MT, int MODE>
cudaError_t launch_t(const TcGemmArgs& a, dim3 grid, cudaStream_t s) {
  auto kern = k_qgemm_tc<FMT, MT, MODE>;
  constexpr size_t smem = tc_smem_bytes<FMT, MT>();
  static bool opted[64] = {};
  const cudaError_t e = opt_in_smem(kern, (int)smem, opted);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, dim3(kThreads), smem, s, a);
}

template <int FMT, int MODE>
cudaError_t launch_mt(const TcGemmArgs& a, dim3 grid, cudaStream_t s) {
  return a.mt == 2 ? launch_t<FMT, 2, MODE>(a, grid, s) : launch_t<FMT, 1, MODE>(a, grid, s);
}

bool tile_ok(int tile, int mode) {
  if (tile < 8 || tile % 8 != 0) return false;
  return mode == TC_GATEUP ? tile <= 128 : (tile <= kMaxRows && tile % 16 == 0);
}

}  // namespace

int tc_gateup_feat(int I) {
  const int f = ((I + 7) / 8) * 8;
  return f < 128 ? f : 128;
}

int tc_down_rows(int H) {
  const int r = ((H + 15) / 16) * 16;
  return r < kMaxRows ? r : kMaxRows;
}

int tc_mt_for(int tokens) { return tokens > kTokRows ? 2 : 1; }

int tc_tokens_per_cta(int mt) { return mt * kTokRows; }

cudaError_t encode_tc_weight_maps(TcMaps* m, int fmt, const QW& w, int N, int K, int box_rows) {
  cudaError_t e;
  if (fmt == FMT_INT4_G32) {
    e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.q, K / 2, N, K / 2, 128, box_rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = encode_tmap_2d(&m->scale, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.scale, K / 32, N, K / 16, 8, box_rows);
    if (e != cudaSuccess) return e;
    return encode_tmap_2d(&m->mn, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.mn, K / 32, N, K / 16, 8, box_rows);
  }
  e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.q, K, N, K, 128, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
  m->scale = m->codes;
  m->mn = m->codes;
  return e;
}

cudaError_t encode_tc_x_map(CUtensorMap* m, const uint16_t* x, int rows, int K) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, rows, (uint64_t)K * 2, 64, kTokRows,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_tc_gemm(const TcGemmArgs& a, int row_tiles, int splits, int jobs, cudaStream_t s) {
  if (!tile_ok(a.tile, a.mode)) return cudaErrorInvalidValue;
  if (a.offsets != nullptr && a.Ns > 0 && !tile_ok(a.tile_s, a.mode)) return cudaErrorInvalidValue;
  if (a.mt != 1 && a.mt != 2) return cudaErrorInvalidValue;
  const dim3 grid(row_tiles, a.token_tiles * splits, jobs);
  if (a.fmt == FMT_INT4_G32)
    return a.mode == TC_GATEUP ? launch_mt<FMT_INT4_G32, TC_GATEUP>(a, grid, s)
                               : launch_mt<FMT_INT4_G32, TC_DOWN>(a, grid, s);
  return a.mode == TC_GATEUP ? launch_mt<FMT_INT8_ROW, TC_GATEUP>(a, grid, s)
                             : launch_mt<FMT_INT8_ROW, TC_DOWN>(a, grid, s);
}

unsigned int tc_gemm_fault_flags(bool clear) {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, g_fault_flags, sizeof(v));
  if (clear && v) {
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_fault_flags, &z, sizeof(z));
  }
  return v;
}

}  // namespace moeffn
