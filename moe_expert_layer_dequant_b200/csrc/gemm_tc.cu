// Quantized GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), for
// several token rows per weight matrix (prefill, batched decode, and the
// grouped expert GEMMs of the MoE layer).
//
// Operand roles: the dequantized weights are the MMA's A operand and live in
// TMEM (M = 128 weight rows per tile); the bf16 token rows are B in shared
// memory (N = the CTA's token rows rounded up to 16, at most kTcMaxTok). Each
// weight is dequantized once per CTA straight from registers into TMEM
// (tcgen05.st): no shared-memory round trip for the dequantized tile, and the
// MMA reads only the token tile from shared memory.
//
// Per CTA: two A tiles of 128 weight rows that share every token tile (GATEUP:
// 128 gate rows and the same 128 up rows, so a feature's gate and up sums sit
// in one TMEM lane of two accumulators; DOWN: 256 consecutive output rows),
// one tile of token rows, and the job's K range (or one K split of it).
//
//  warp 0      weight producer: TMA loads of the quantized weight stages (codes
//              in 128-byte swizzled boxes, INT4 group scales and mins), both
//              A tiles;
//  warp 1      allocates TMEM; one thread issues tile 0's tcgen05.mma;
//  warp 2      token producer: TMA loads of the bf16 token tiles (128-byte
//              swizzled, K = 64 per stage), the MMA's B operand, one per A
//              stage slot (the two operands of a stage share one full and
//              one empty barrier);
//  warp 3      one thread issues tile 1's tcgen05.mma (the two accumulators
//              are independent; issuing from two threads halves the per-stage
//              issue time); A and B slots are released once both issuers'
//              tcgen05.commit have arrived;
//  warps 4-19  dequantize, in two sets of eight taking the A stages (K = 64)
//              in turn: a thread owns one weight row of one A tile and turns
//              the 64 codes of two quantization groups into bf16 (RNE of the
//              exact fp32 value q * scale + min), stored to its TMEM lane (32
//              columns of bf16 pairs); one thread per set waits on and
//              arrives at the mbarriers for the set, whose warps meet at a
//              named barrier before and after the stage; then, as the
//              epilogue, read the accumulators (tcgen05.ld) and write the
//              outputs.
//
// TMEM columns: accumulator of A tile t at [t * ntile, (t + 1) * ntile); a ring
// of A stages (two K groups each: 32 columns per A tile) after them; the
// ring depth SA (2 to 7) is what the accumulators leave. Waits
// suspend the waiting thread (mbarrier.try_wait) rather than spin, so the
// producer and MMA threads take no issue slots from the dequantizing warps.
// Modes: GATEUP writes bf16(act(gate) * up); DOWN writes fp32 partial sums
// d[split][slot][row] that the layer tails combine. INT8-row weights enter the
// MMA as their exact integer codes and are scaled per row in the epilogue.
#include "gemm_tc.cuh"
#include "launch.cuh"
#include "sync.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace moeffn {

namespace {

constexpr int kTilesA = 2;                   // A tiles per CTA
constexpr int kDqWarps = 16;                 // warps 4..19, two sets of 8
constexpr int kThreads = 32 * (4 + kDqWarps);
constexpr int kSW = 3;                       // quantized weight stages
constexpr int kBRingBytes = 64 * 1024;      // token stages: one per A stage slot (SA * ntile * 128 bytes)
constexpr int kTmemCols = 512;
constexpr int kAStageCols = 32 * kTilesA;    // two K groups (64 bf16 = 32 columns) per A tile

template <int FMT>
struct TcFmt;
template <>
struct TcFmt<FMT_INT4_G32> {
  static constexpr int kKTile = 256;                        // codes per weight stage row (128 bytes)
  static constexpr int kGroups = kKTile / 32;               // K groups (A stages) per weight stage
  static constexpr int kCodeBytes = kTcRowsA * 128;
  static constexpr int kScaleBytes = kTcRowsA * 16;         // 8 fp16 per row
  static constexpr int kTileBytes = kCodeBytes + 2 * kScaleBytes;
  static constexpr int kStageBytes = kTilesA * kTileBytes;
};
template <>
struct TcFmt<FMT_INT8_ROW> {
  static constexpr int kKTile = 128;
  static constexpr int kGroups = kKTile / 32;
  static constexpr int kCodeBytes = kTcRowsA * 128;
  static constexpr int kScaleBytes = 0;
  static constexpr int kTileBytes = kCodeBytes;
  static constexpr int kStageBytes = kTilesA * kTileBytes;
};

template <>
struct TcFmt<FMT_Q4K> {
  static constexpr int kKTile = Q4K::kBlock;                // one super-block per row and stage
  static constexpr int kGroups = kKTile / 32;
  static constexpr int kCodeBytes = kTcRowsA * Q4K::kBytes; // unswizzled rows of 144 bytes
  static constexpr int kScaleBytes = 0;
  static constexpr int kTileBytes = kCodeBytes;
  static constexpr int kStageBytes = kTilesA * kTileBytes;
};

template <int FMT>
constexpr size_t tc_smem_bytes() {
  return 1024 /*align slack*/ + 1024 /*barriers*/ + (size_t)kSW * TcFmt<FMT>::kStageBytes + kBRingBytes;
}
static_assert(tc_smem_bytes<FMT_INT4_G32>() <= 232448, "shared memory");
static_assert(tc_smem_bytes<FMT_INT8_ROW>() <= 232448, "shared memory");
static_assert(tc_smem_bytes<FMT_Q4K>() <= 232448, "shared memory");
static_assert(TcFmt<FMT_INT4_G32>::kStageBytes % 1024 == 0 && TcFmt<FMT_INT8_ROW>::kStageBytes % 1024 == 0 &&
                  TcFmt<FMT_Q4K>::kStageBytes % 1024 == 0,
              "stage bases stay 1024-byte aligned (128-byte swizzle)");

struct Job {
  const TcMaps* m0;
  const TcMaps* m1;
  const CUtensorMap* xmap;
  const __half* rs0;
  const __half* rs1;
  int N, K, ntok, slot0;
  bool shared, valid;
};

__device__ __forceinline__ Job decode_job(const TcGemmArgs& a) {
  Job j{};
  j.valid = true;
  const int z = blockIdx.y;
  if (a.offsets == nullptr) {
    j.m0 = &a.w0; j.m1 = &a.w1; j.xmap = &a.xmap; j.rs0 = a.rscale0; j.rs1 = a.rscale1;
    j.N = a.N; j.K = a.K; j.ntok = a.M;
  } else if (z < a.routed_jobs) {
    if (z >= *a.n_union) { j.valid = false; return j; }
    const int e = a.union_list[z];
    j.m0 = a.tab0 + e;
    j.m1 = a.tab1 != nullptr ? a.tab1 + e : nullptr;
    j.xmap = &a.xmap;
    j.N = a.N; j.K = a.K;
    j.slot0 = a.offsets[e];
    j.ntok = a.offsets[e + 1] - j.slot0;
  } else {
    j.m0 = &a.s0; j.m1 = &a.s1; j.xmap = &a.xmap_s;
    j.N = a.Ns; j.K = a.Ks; j.ntok = a.M; j.shared = true;
  }
  if (a.mode == TC_DOWN) j.m1 = j.m0;   // the second A tile is 128 rows further down the same matrix
  return j;
}

__device__ __forceinline__ uint32_t lds_u16(uint32_t addr) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}

// ---- dequantization of one K group (32 weights) of one row ---------------
// Output: 16 bf16 pairs, element 2c in the low half of o[c] (the TMEM layout
// of the MMA's A operand).

// INT4: group g of the stage row is 16-byte chunk g of the 128-byte swizzled
// row (stored at chunk g ^ (r % 8)); code i of a word sits at bits 4i..4i+3.
// The magic conversion leaves the code of bits 4i scaled by 16^(i%4): the
// scale carries the inverse power of two (exact). w = q * s + m in fp32 is
// exact (q * s has at most 15 significant bits, both terms are multiples of
// 2^-24 and |w| < 1), then rounded once to bf16.
__device__ __forceinline__ void dq_group_int4(uint32_t tile, int r, int g, uint32_t (&o)[16]) {
  using F = TcFmt<FMT_INT4_G32>;
  const uint4 cw = lds_u128(tile + r * 128 + (((g ^ (r & 7)) & 7) << 4));
  const float s = __half2float(__ushort_as_half((unsigned short)lds_u16(tile + F::kCodeBytes + r * 16 + g * 2)));
  const float m =
      __half2float(__ushort_as_half((unsigned short)lds_u16(tile + F::kCodeBytes + F::kScaleBytes + r * 16 + g * 2)));
  const uint32_t mg = kMagic, m0 = 0x000Fu, m1 = 0x00F0u, m2 = 0x0F00u, m3 = 0xF000u;
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
    o[4 * q + 0] = pack_bf16x2(c01.x, c01.y);
    o[4 * q + 1] = pack_bf16x2(c23.x, c23.y);
    o[4 * q + 2] = pack_bf16x2(c45.x, c45.y);
    o[4 * q + 3] = pack_bf16x2(c67.x, c67.y);
  }
}

// Q4_K: A stage a (0..3) of a weight stage is code run a of the row's block:
// 32 bytes whose low nibbles are the stage's K elements 0..31 (sub-block 2a,
// into o0) and whose high nibbles are elements 32..63 (sub-block 2a + 1, into
// o1). Each value is fmaf(q, d * scale, -dmin * min), the exact weight rounded
// once to fp32, then rounded to bf16. The masks pick the nibbles of bytes 0
// and 1 (lo) or of their high halves (hi) in place, so the scale is divided by
// the nibble's place value (exact: a power of two).
__device__ __forceinline__ void dq_run_q4k(uint32_t tile, int r, int a, uint32_t (&o0)[16], uint32_t (&o1)[16]) {
  const uint32_t row = tile + r * Q4K::kBytes;
  const uint4 hdr = lds_u128(row);
  const uint4 ca = lds_u128(row + 16 + 32 * a), cb = lds_u128(row + 32 + 32 * a);
  float sl, ml, sh, mh;
  Q4K::scale_min(hdr, 2 * a, sl, ml);
  Q4K::scale_min(hdr, 2 * a + 1, sh, mh);
  const uint32_t mg = kMagic;
  const float2 sub = make_float2(-kMagicF, -kMagicF);
  const float2 lo_s = make_float2(sl, sl * 0.00390625f), lo_m = make_float2(ml, ml);
  const float2 hi_s = make_float2(sh * 0.0625f, sh * 0.000244140625f), hi_m = make_float2(mh, mh);
  const uint32_t words[8] = {ca.x, ca.y, ca.z, ca.w, cb.x, cb.y, cb.z, cb.w};
#pragma unroll
  for (int q = 0; q < 8; ++q) {   // word q: elements 4q..4q+3 of both sub-blocks
    const uint32_t w = words[q], h = w >> 16;
    float2 l01 = make_float2(__uint_as_float(and_or(w, 0x000Fu, mg)), __uint_as_float(and_or(w, 0x0F00u, mg)));
    float2 l23 = make_float2(__uint_as_float(and_or(h, 0x000Fu, mg)), __uint_as_float(and_or(h, 0x0F00u, mg)));
    float2 h01 = make_float2(__uint_as_float(and_or(w, 0x00F0u, mg)), __uint_as_float(and_or(w, 0xF000u, mg)));
    float2 h23 = make_float2(__uint_as_float(and_or(h, 0x00F0u, mg)), __uint_as_float(and_or(h, 0xF000u, mg)));
    l01 = __ffma2_rn(__fadd2_rn(l01, sub), lo_s, lo_m);
    l23 = __ffma2_rn(__fadd2_rn(l23, sub), lo_s, lo_m);
    h01 = __ffma2_rn(__fadd2_rn(h01, sub), hi_s, hi_m);
    h23 = __ffma2_rn(__fadd2_rn(h23, sub), hi_s, hi_m);
    o0[2 * q] = pack_bf16x2(l01.x, l01.y);
    o0[2 * q + 1] = pack_bf16x2(l23.x, l23.y);
    o1[2 * q] = pack_bf16x2(h01.x, h01.y);
    o1[2 * q + 1] = pack_bf16x2(h23.x, h23.y);
  }
}

// INT8: group g is chunks 2g, 2g + 1 of the 128-byte swizzled row (32 signed
// codes), entered as exact bf16 integers; the row scale is applied in the
// epilogue.
__device__ __forceinline__ void dq_group_int8(uint32_t tile, int r, int g, uint32_t (&o)[16]) {
  const uint32_t mg = kMagic;
  const float2 sub = make_float2(-(kMagicF + 128.0f), -(kMagicF + 128.0f));
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int chunk = 2 * g + h;
    const uint4 cw = lds_u128(tile + r * 128 + (((chunk ^ (r & 7)) & 7) << 4));
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
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
      o[8 * h + 2 * q] = pack_bf16x2(v01.x, v01.y);
      o[8 * h + 2 * q + 1] = pack_bf16x2(v23.x, v23.y);
    }
  }
}

template <int FMT, int MODE>
__global__ void __launch_bounds__(kThreads, 1) k_qgemm_tc(const __grid_constant__ TcGemmArgs a) {
  using F = TcFmt<FMT>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  pdl_wait();
  const Job job = decode_job(a);
  if (!job.valid) return;
  const int ntile = a.ntile;
  // grid.z runs over token tiles (slowest) and K splits: every job's first
  // token tile is scheduled before any later one, so the tiles past an
  // expert's token count (which exit at once) come last, in the wave tail.
  const int splits = (int)gridDim.z / a.token_tiles;
  const int tt = blockIdx.z / splits, split = blockIdx.z % splits;
  const int t0 = tt * ntile;
  if (t0 >= job.ntok) return;
  // Weight rows of the CTA: GATEUP features f0..f0+127 of gate (tile 0) and
  // up (tile 1); DOWN rows r0..r0+255 (tiles 0 and 1).
  const int row0 = blockIdx.x * (MODE == TC_GATEUP ? kTcGateUpFeat : kTcDownRows);
  if (row0 >= job.N) return;
  const int row1 = MODE == TC_GATEUP ? row0 : row0 + kTcRowsA;
  const int tiles = (MODE == TC_DOWN && row1 >= job.N) ? 1 : 2;   // a DOWN tile entirely past the end is skipped
  const int k0 = split * a.ks_len;
  if (k0 >= job.K) return;
  const int klen = min(a.ks_len, job.K - k0);     // a multiple of the weight stage K
  const int nA = klen / 64;                         // A stages (two K groups each)
  const int nW = klen / F::kKTile;                  // weight stages
  const int tn = min(ntile, job.ntok - t0);         // valid token rows
  const int nmma = (tn + 15) & ~15;                 // MMA N
  const int SA = min(8, (kTmemCols - kTilesA * ntile) / kAStageCols);   // A ring depth (2..7)
  const uint32_t a_col0 = (uint32_t)(kTilesA * ntile);

  // ---- shared memory carve (1024-byte aligned operand tiles) -------------
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_addr(smem_raw));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase);
  uint64_t* w_full = bars;
  uint64_t* w_empty = w_full + kSW;
  uint64_t* full = w_empty + kSW;     // [8] A stage dequantized and its token tile landed
  uint64_t* empty = full + 8;         // [8] both MMA issuers done with the slot
  uint64_t* acc_full = empty + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + 512);
  volatile int* set_dead = reinterpret_cast<volatile int*>(gbase + 520);   // [2] a set's waiter gave up
  const uint32_t w_base = base + 1024;
  const uint32_t b_base = w_base + kSW * F::kStageBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kSW; ++i) { mbar_init(&w_full[i], 1); mbar_init(&w_empty[i], 2); }
    // full: one arrival per dequantizing set plus the token producer's
    // expect_tx arrival (and its bytes); empty: one commit per MMA issuer.
    for (int i = 0; i < 8; ++i) { mbar_init(&full[i], 2); mbar_init(&empty[i], 2); }
    set_dead[0] = set_dead[1] = 0;
    mbar_init(acc_full, 2);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
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
    if (lane == 0 && SA >= 2) {
      const uint32_t tx = (uint32_t)tiles * F::kTileBytes;
      int issued = 0;
      for (int w = 0; w < nW; ++w, ++issued) {
        const int slot = w % kSW, use = w / kSW;
        if (use > 0 && !mbar_wait(&w_empty[slot], (use - 1) & 1)) break;
        uint8_t* gst = gbase + (w_base - base) + slot * F::kStageBytes;
        mbar_arrive_expect_tx(&w_full[slot], tx);
        const int kc = k0 + w * F::kKTile;                  // first K element of the stage
        const int cx = (FMT == FMT_INT4_G32) ? kc / 2 : (FMT == FMT_Q4K) ? kc / Q4K::kBlock * Q4K::kBytes : kc;  // byte column
        for (int t = 0; t < tiles; ++t) {
          const TcMaps* mp = t == 0 ? job.m0 : job.m1;
          const int rw = t == 0 ? row0 : row1;
          uint8_t* dst = gst + t * F::kTileBytes;
          tma_load_2d(dst, &mp->codes, cx, rw, &w_full[slot]);
          if (FMT == FMT_INT4_G32) {
            tma_load_2d(dst + F::kCodeBytes, &mp->scale, kc / 32, rw, &w_full[slot]);
            tma_load_2d(dst + F::kCodeBytes + F::kScaleBytes, &mp->mn, kc / 32, rw, &w_full[slot]);
          }
        }
      }
      // No copy is left in flight when the CTA exits (after a timed-out wait
      // too): the last stages issued have landed.
      for (int w = max(0, issued - kSW); w < issued; ++w) mbar_wait(&w_full[w % kSW], (w / kSW) & 1);
    }
  } else if (warp == 2) {
    // ---------------- token producer ----------------
    if (lane == 0 && SA >= 2) {
      int issued = 0;
      for (int b = 0; b < nA; ++b, ++issued) {
        const int slot = b % SA, use = b / SA;
        if (use > 0 && !mbar_wait(&empty[slot], (use - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[slot], (uint32_t)ntile * 128u);
        uint8_t* dst = gbase + (b_base - base) + slot * ntile * 128;
        tma_load_2d(dst, job.xmap, k0 + b * 64, row_tok, &full[slot]);
      }
      for (int b = max(0, issued - SA); b < issued; ++b) mbar_wait(&full[b % SA], (b / SA) & 1);
    }
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers: warp 1 for A tile 0, warp 3 for tile 1 ----
    // The two accumulators are independent, so each tile's MMAs come from its
    // own thread (on its own SM sub-partition); slots are released when both
    // threads' commits have arrived.
    const int tl = warp == 1 ? 0 : 1;
    if (lane == 0 && SA >= 2) {
      const uint32_t idesc = idesc_bf16_f32(kTcRowsA, nmma);
      for (int s = 0; s < nA; ++s) {
        const int slot = s % SA;
        if (!mbar_wait(&full[slot], (s / SA) & 1)) break;
        tc_fence_after();
        const uint64_t bd = umma_desc_sw128(b_base + slot * ntile * 128);
        const uint32_t acol = tmem + a_col0 + (uint32_t)(slot * kAStageCols);
        if (tl < tiles) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ts(tmem + (uint32_t)(tl * ntile), acol + (uint32_t)(tl * 32 + kk * 8), bd + 2 * kk, idesc,
                         (s | kk) != 0);
        }
        umma_commit(&empty[slot]);
      }
      umma_commit(acc_full);
      mbar_wait(acc_full, 0);   // every MMA has completed before TMEM is freed
    }
  } else if (warp >= 4) {
    // ---------------- dequantize (warps 4-19), then epilogue ----------------
    const int i = warp - 4;
    const int set = i >> 3, q = i & 3, t = (i >> 2) & 1;   // K-group parity, lane quarter, A tile
    const int r = 32 * q + lane;                           // weight row of the A tile
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    // One thread per set (lane 0 of the set's first warp) waits on the
    // barriers and arrives for the set; the set's eight warps meet at a named
    // barrier before and after the dequantization.
    const bool waiter = (i & 7) == 0 && lane == 0;
    bool dead = SA < 2;
    for (int s = set; s < nA && !dead; s += 2) {
      const int slot = s % SA, use = s / SA;
      constexpr int kAPerW = F::kGroups / 2;                           // A stages per weight stage
      const int w = s / kAPerW, g = 2 * (s % kAPerW), ws = w % kSW;
      if (waiter) {
        bool ok = true;
        if (s % kAPerW == set) ok = mbar_wait(&w_full[ws], (w / kSW) & 1);   // first A stage of the weight stage for this set
        if (ok && use > 0) ok = mbar_wait(&empty[slot], (use - 1) & 1);
        if (!ok) set_dead[set] = 1;
      }
      named_sync(1 + set, 256);
      if (set_dead[set] != 0) { dead = true; break; }   // the whole set leaves together
      tc_fence_after();
      if (t < tiles) {
        uint32_t o0[16], o1[16];
        const uint32_t tile = w_base + ws * F::kStageBytes + t * F::kTileBytes;
        if (FMT == FMT_INT4_G32) { dq_group_int4(tile, r, g, o0); dq_group_int4(tile, r, g + 1, o1); }
        else if (FMT == FMT_Q4K) dq_run_q4k(tile, r, g / 2, o0, o1);
        else { dq_group_int8(tile, r, g, o0); dq_group_int8(tile, r, g + 1, o1); }
        const uint32_t ta = tmem + lane_base + a_col0 + (uint32_t)(slot * kAStageCols + t * 32);
        tmem_st16(ta, o0);
        tmem_st16(ta + 16, o1);
        tmem_wait_st();
      }
      tc_fence_before();
      named_sync(1 + set, 256);
      if (waiter) {
        mbar_arrive(&full[slot]);
        if (s % kAPerW == kAPerW - 2 + set) mbar_arrive(&w_empty[ws]);   // this set's last A stage of the weight stage
      }
    }
    // Epilogue: TMEM lanes = weight rows, columns = token rows of the tile.
    if (!dead && !mbar_wait(acc_full, 0)) dead = true;
    dead = __any_sync(0xffffffffu, dead);   // TMEM loads are warp-collective
    tc_fence_after();
    const int share = i >> 2;               // 4 warps per lane quarter share the columns
    const int nchunks = nmma / 16;
    if (!dead && MODE == TC_GATEUP) {
      const int f = row0 + r;
      const bool fvalid = f < job.N;
      float sg = 1.f, su = 1.f;
      if (FMT == FMT_INT8_ROW && fvalid) {
        sg = __half2float(job.rs0[f]);
        su = __half2float(job.rs1[f]);
      }
      uint16_t* out = job.shared ? a.out_act_s : a.out_act;
      for (int c = share; c < nchunks; c += 4) {
        float gv[16], uv[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(16 * c), gv);
        tmem_ld16(tmem + lane_base + (uint32_t)(ntile + 16 * c), uv);
        if (fvalid) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = 16 * c + j;
            if (tok < tn)
              out[(size_t)(row_tok + tok) * job.N + f] = float_to_bf16_bits(gated_act(gv[j] * sg, uv[j] * su, a.act));
          }
        }
      }
    } else if (!dead) {
      float* dout = job.shared ? a.out_d_s : a.out_d;
      const int nslots = job.shared ? a.M : a.slots;
      for (int idx = share; idx < tiles * nchunks; idx += 4) {
        const int tl = idx % tiles, c = idx / tiles;
        float v[16];
        tmem_ld16(tmem + lane_base + (uint32_t)(tl * ntile + 16 * c), v);
        const int row = (tl == 0 ? row0 : row1) + r;
        if (row < job.N) {
          const float sd = FMT == FMT_INT8_ROW ? __half2float(job.rs0[row]) : 1.f;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int tok = 16 * c + j;
            if (tok < tn) dout[((size_t)split * nslots + row_tok + tok) * job.N + row] = v[j] * sd;
          }
        }
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int FMT, int MODE>
cudaError_t launch_t(const TcGemmArgs& a, dim3 grid, cudaStream_t s) {
  auto kern = k_qgemm_tc<FMT, MODE>;
  constexpr size_t smem = tc_smem_bytes<FMT>();
  static bool opted[64] = {};
  const cudaError_t e = opt_in_smem(kern, (int)smem, opted);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, dim3(kThreads), smem, s, a);
}

}  // namespace

int tc_ntile_for(int tokens) {
  if (tokens < 1) tokens = 1;
  const int tiles = (tokens + kTcMaxTok - 1) / kTcMaxTok;
  const int per = (tokens + tiles - 1) / tiles;
  return (per + 15) & ~15;
}

cudaError_t encode_tc_weight_maps(TcMaps* m, int fmt, const QW& w, int N, int K) {
  cudaError_t e;
  if (fmt == FMT_INT4_G32) {
    e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.q, K / 2, N, K / 2, 128, kTcRowsA,
                       CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = encode_tmap_2d(&m->scale, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.scale, K / 32, N, K / 16, 8, kTcRowsA);
    if (e != cudaSuccess) return e;
    return encode_tmap_2d(&m->mn, CU_TENSOR_MAP_DATA_TYPE_UINT16, w.mn, K / 32, N, K / 16, 8, kTcRowsA);
  }
  if (fmt == FMT_Q4K) {   // one 144-byte block per row and stage, unswizzled
    const uint64_t rb = (uint64_t)K / Q4K::kBlock * Q4K::kBytes;
    e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.q, rb, N, rb, Q4K::kBytes, kTcRowsA);
    m->scale = m->codes;
    m->mn = m->codes;
    return e;
  }
  e = encode_tmap_2d(&m->codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.q, K, N, K, 128, kTcRowsA,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  m->scale = m->codes;
  m->mn = m->codes;
  return e;
}

cudaError_t encode_tc_x_map(CUtensorMap* m, const uint16_t* x, int rows, int K, int ntile) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, rows, (uint64_t)K * 2, 64, ntile,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_tc_gemm(const TcGemmArgs& a, int row_tiles, int splits, int jobs, cudaStream_t s) {
  if (a.ntile < 16 || a.ntile > kTcMaxTok || a.ntile % 16 != 0) return cudaErrorInvalidValue;
  if (a.ks_len <= 0 || a.ks_len % tc_k_tile(a.fmt) != 0) return cudaErrorInvalidValue;
  const dim3 grid(row_tiles, jobs, a.token_tiles * splits);
  if (a.fmt == FMT_INT4_G32)
    return a.mode == TC_GATEUP ? launch_t<FMT_INT4_G32, TC_GATEUP>(a, grid, s) : launch_t<FMT_INT4_G32, TC_DOWN>(a, grid, s);
  if (a.fmt == FMT_Q4K)
    return a.mode == TC_GATEUP ? launch_t<FMT_Q4K, TC_GATEUP>(a, grid, s) : launch_t<FMT_Q4K, TC_DOWN>(a, grid, s);
  return a.mode == TC_GATEUP ? launch_t<FMT_INT8_ROW, TC_GATEUP>(a, grid, s) : launch_t<FMT_INT8_ROW, TC_DOWN>(a, grid, s);
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
