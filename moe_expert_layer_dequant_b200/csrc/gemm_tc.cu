// Quantized GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), for
// several token rows per weight matrix (prefill, batched decode, and the
// grouped expert GEMMs of the MoE layer).
//
// Swap-AB: the MMA's M dimension (128) runs over weight rows, its N dimension
// over tokens (NT = 16..256), so a handful of tokens per expert still fills
// the instruction. Per CTA: one tile of weight rows x one tile of tokens x the
// job's K range (or one K split of it).
//
//  warp 0      weight producer: TMA loads of the quantized weight stages
//              (codes in 128-byte swizzled boxes, INT4 group scales and mins);
//  warp 2      token producer: TMA loads of the bf16 token tiles (128-byte
//              swizzled, the MMA's B operand);
//  warp 1      allocates the TMEM accumulator and issues tcgen05.mma (one
//              thread), releasing operand slots with tcgen05.commit;
//  warps 4-19  dequantize, in two groups of 8 warps taking alternate K atoms:
//              two threads per weight row each write 32 bf16 weights of the
//              atom (w = RNE(q * scale + min), exact in fp32 before the
//              rounding) into the swizzled canonical layout the MMA reads;
//  warps 4-7   then, as the epilogue, read TMEM (warp w%4 sees lanes
//              32*(w%4)..+31) and write the outputs.
//
// Modes: GATEUP stacks 64 gate rows and the same 64 up rows in one 128-row A
// tile; the epilogue pairs them (through shared memory) into
// bf16(act(gate) * up). DOWN writes fp32 partial sums d[split][slot][row]
// that the layer tails combine. INT8-row weights enter the MMA as their exact
// integer codes and are scaled per row in the epilogue.
#include "gemm_tc.cuh"
#include "launch.cuh"
#include "sync.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace moeffn {

namespace {

constexpr int kDqGroups = 2;            // dequant groups, taking alternate K atoms
constexpr int kDqGroupWarps = 8;        // warps per group: two threads per weight row
constexpr int kDqWarps = kDqGroups * kDqGroupWarps;   // warps 4..19
constexpr int kThreads = 32 * (4 + kDqWarps);
constexpr int kAtomBytes = 128 * 128;   // 128 rows x 64 bf16

template <int FMT>
struct TcFmt;
template <>
struct TcFmt<FMT_INT4_G32> {
  static constexpr int kKTile = 256;      // codes per weight stage row (128 bytes)
  static constexpr int kAtoms = 4;        // K atoms of 64 per stage
  static constexpr int kCodeBytes = 128 * 128;
  static constexpr int kScaleBytes = 128 * 16;
  static constexpr int kStageBytes = kCodeBytes + 2 * kScaleBytes;
};
template <>
struct TcFmt<FMT_INT8_ROW> {
  static constexpr int kKTile = 128;
  static constexpr int kAtoms = 2;
  static constexpr int kCodeBytes = 128 * 128;
  static constexpr int kScaleBytes = 0;
  static constexpr int kStageBytes = kCodeBytes;
};

template <int NT>
struct TcTile {
  static constexpr int kSB = NT >= 256 ? 3 : 4;                 // B (token) atoms
  static constexpr int kSW = NT <= 128 ? 4 : 2;                 // quantized weight stages
  static constexpr int kSA = NT <= 32 ? 8 : (NT <= 64 ? 6 : 4); // bf16 A atoms
  static constexpr int kBBytes = NT * 128;
  static constexpr uint32_t kTmemCols = NT < 32 ? 32u : (uint32_t)NT;
};

template <int FMT, int NT>
__host__ __device__ constexpr size_t tc_smem_bytes() {
  return 1024 /*align slack*/ + 1024 /*barriers*/ + (size_t)TcTile<NT>::kSW * TcFmt<FMT>::kStageBytes +
         (size_t)TcTile<NT>::kSA * kAtomBytes + (size_t)TcTile<NT>::kSB * TcTile<NT>::kBBytes;
}

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
  const int z = blockIdx.z;
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
  return j;
}

// ---- dequantization of one K atom (64 weights) of one row into the A tile ----

// INT4: half hf of atom j is group g = 2j + hf of the stage row (one 16-byte
// chunk of the 128-byte swizzled row, 32 codes); w = q * s + m in fp32
// (exact), rounded to bf16, written as chunks 4hf..4hf+3 of the atom row.
__device__ __forceinline__ void dequant_half_int4(uint32_t wq, int r, int j, int hf, uint32_t a_atom) {
  const uint32_t code_row = wq + r * 128;
  const int g = 2 * j + hf;
  const uint32_t sw = lds_u32(wq + TcFmt<FMT_INT4_G32>::kCodeBytes + r * 16 + (g >> 1) * 4);
  const uint32_t mw = lds_u32(wq + TcFmt<FMT_INT4_G32>::kCodeBytes + TcFmt<FMT_INT4_G32>::kScaleBytes + r * 16 + (g >> 1) * 4);
  const float s = __half2float(__ushort_as_half((unsigned short)((sw >> ((g & 1) * 16)) & 0xFFFFu)));
  const float m = __half2float(__ushort_as_half((unsigned short)((mw >> ((g & 1) * 16)) & 0xFFFFu)));
  const uint4 cw = lds_u128(code_row + (((g ^ (r & 7)) & 7) << 4));
  const uint32_t arow = a_atom + r * 128;
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
    sts_u128(arow + ((chunk ^ (r & 7)) << 4), out);
  }
}

// INT8: half hf of atom j is input chunks 4j+2hf, 4j+2hf+1 (32 signed codes)
// as exact bf16 integers; the row scale is applied in the epilogue.
__device__ __forceinline__ void dequant_half_int8(uint32_t wq, int r, int j, int hf, uint32_t a_atom) {
  const uint32_t code_row = wq + r * 128;
  const uint32_t arow = a_atom + r * 128;
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
    sts_u128(arow + ((ch0 ^ (r & 7)) << 4), make_uint4(packed[0], packed[1], packed[2], packed[3]));
    sts_u128(arow + ((ch1 ^ (r & 7)) << 4), make_uint4(packed[4], packed[5], packed[6], packed[7]));
  }
}

template <int FMT, int NT, int MODE>
__global__ void __launch_bounds__(kThreads, 1) k_qgemm_tc(const __grid_constant__ TcGemmArgs a) {
  using F = TcFmt<FMT>;
  using T = TcTile<NT>;
  constexpr int ROWS = (MODE == TC_GATEUP) ? 64 : 128;   // output rows of the tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  pdl_wait();
  const Job job = decode_job(a);
  if (!job.valid) return;
  const int tt = blockIdx.y % a.token_tiles, split = blockIdx.y / a.token_tiles;
  const int t0 = tt * NT;
  if (t0 >= job.ntok) return;
  const int n0 = blockIdx.x * ROWS;
  if (n0 >= job.N) return;
  const int k0 = split * a.ks_len;
  if (k0 >= job.K) return;
  const int klen = min(a.ks_len, job.K - k0);
  const int nk = klen / 64;                     // K atoms (klen is a multiple of the stage K)
  const int tn = min(NT, job.ntok - t0);        // valid token columns

  // ---- shared memory carve (1024-byte aligned operand tiles) -------------
  const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
  uint8_t* const gbase = smem_raw + (base - smem_addr(smem_raw));
  uint64_t* bars = reinterpret_cast<uint64_t*>(gbase);
  uint64_t* wq_full = bars;
  uint64_t* wq_empty = wq_full + T::kSW;
  uint64_t* a_full = wq_empty + T::kSW;
  uint64_t* a_empty = a_full + T::kSA;
  uint64_t* b_full = a_empty + T::kSA;
  uint64_t* b_empty = b_full + T::kSB;
  uint64_t* acc_full = b_empty + T::kSB;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + 512);
  const uint32_t wq_base = base + 1024;
  const uint32_t a_base = wq_base + T::kSW * F::kStageBytes;
  const uint32_t b_base = a_base + T::kSA * kAtomBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < T::kSW; ++i) { mbar_init(&wq_full[i], 1); mbar_init(&wq_empty[i], kDqWarps); }
    for (int i = 0; i < T::kSA; ++i) { mbar_init(&a_full[i], kDqGroupWarps); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < T::kSB; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
    mbar_init(acc_full, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, T::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  const int row_tok = job.slot0 + t0;   // first B row (token or slot) of the tile

  if (warp == 0) {
    // ---------------- weight producer ----------------
    // Runs up to kSW stages ahead of the dequantizers, independently of the
    // token tiles, so the weight stream never waits on MMA progress.
    if (lane == 0) {
      const int nw = nk / F::kAtoms;
      for (int w = 0; w < nw; ++w) {
        const int slot = w % T::kSW, use = w / T::kSW;
        if (use > 0 && !mbar_wait_spin(&wq_empty[slot], (use - 1) & 1)) break;
        const uint32_t st = wq_base + slot * F::kStageBytes;
        uint8_t* gst = gbase + (st - base);
        mbar_arrive_expect_tx(&wq_full[slot], F::kStageBytes);
        const int kc = k0 + w * F::kKTile;                 // first K element of the stage
        const int cx = (FMT == FMT_INT4_G32) ? kc / 2 : kc; // byte column of the codes
        if (MODE == TC_GATEUP) {
          tma_load_2d(gst, &job.m0->codes, cx, n0, &wq_full[slot]);
          tma_load_2d(gst + 64 * 128, &job.m1->codes, cx, n0, &wq_full[slot]);
          if (FMT == FMT_INT4_G32) {
            uint8_t* gs = gst + F::kCodeBytes;
            tma_load_2d(gs, &job.m0->scale, kc / 32, n0, &wq_full[slot]);
            tma_load_2d(gs + 64 * 16, &job.m1->scale, kc / 32, n0, &wq_full[slot]);
            tma_load_2d(gs + F::kScaleBytes, &job.m0->mn, kc / 32, n0, &wq_full[slot]);
            tma_load_2d(gs + F::kScaleBytes + 64 * 16, &job.m1->mn, kc / 32, n0, &wq_full[slot]);
          }
        } else {
          tma_load_2d(gst, &job.m0->codes, cx, n0, &wq_full[slot]);
          if (FMT == FMT_INT4_G32) {
            uint8_t* gs = gst + F::kCodeBytes;
            tma_load_2d(gs, &job.m0->scale, kc / 32, n0, &wq_full[slot]);
            tma_load_2d(gs + F::kScaleBytes, &job.m0->mn, kc / 32, n0, &wq_full[slot]);
          }
        }
      }
    }
  } else if (warp == 2) {
    // ---------------- token-tile producer ----------------
    if (lane == 0) {
      for (int k = 0; k < nk; ++k) {
        const int slot = k % T::kSB, use = k / T::kSB;
        if (use > 0 && !mbar_wait_spin(&b_empty[slot], (use - 1) & 1)) break;
        mbar_arrive_expect_tx(&b_full[slot], T::kBBytes);
        tma_load_2d(gbase + (b_base - base) + slot * T::kBBytes, job.xmap, k0 + k * 64, row_tok, &b_full[slot]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, NT);
      bool dead = false;
      for (int k = 0; k < nk; ++k) {
        const int as = k % T::kSA, bs = k % T::kSB;
        if (!mbar_wait_spin(&a_full[as], (k / T::kSA) & 1) || !mbar_wait_spin(&b_full[bs], (k / T::kSB) & 1)) {
          dead = true;
          break;
        }
        tc_fence_after();
        const uint64_t ad = umma_desc_sw128(a_base + as * kAtomBytes);
        const uint64_t bd = umma_desc_sw128(b_base + bs * T::kBBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)   // 4 x K=16 (32 bytes) inside the 128-byte swizzled row
          umma_bf16(tmem, ad + 2 * kk, bd + 2 * kk, idesc, (k | kk) != 0);
        umma_commit(&a_empty[as]);
        umma_commit(&b_empty[bs]);
      }
      if (!dead) umma_commit(acc_full);
    }
  } else if (warp >= 4) {
    // ---------------- dequantize (warps 4-19), then epilogue (warps 4-7) ----------------
    // Two groups of 8 warps take alternate K atoms, so that one group's store
    // drain and barrier release overlap the other's conversion. Every A slot
    // belongs to one group (the ring depth is even).
    const int grp = (warp - 4) / kDqGroupWarps;
    const int tg = (warp - 4 - grp * kDqGroupWarps) * 32 + lane;
    const int r = tg & 127, hf = tg >> 7;   // weight row of the A tile, half of the atom row
    bool dead = false;
    for (int k = grp; k < nk; k += kDqGroups) {
      const int w = k / F::kAtoms, j = k % F::kAtoms, ws = w % T::kSW;
      const int as = k % T::kSA, ause = k / T::kSA;
      if (!dead && j < kDqGroups && !mbar_wait_spin(&wq_full[ws], (w / T::kSW) & 1)) dead = true;
      if (!dead && ause > 0 && !mbar_wait_spin(&a_empty[as], (ause - 1) & 1)) dead = true;
      if (!dead) {
        const uint32_t wq = wq_base + ws * F::kStageBytes;
        if (FMT == FMT_INT4_G32) dequant_half_int4(wq, r, j, hf, a_base + as * kAtomBytes);
        else dequant_half_int8(wq, r, j, hf, a_base + as * kAtomBytes);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&a_full[as]);
        if (j >= F::kAtoms - kDqGroups) mbar_arrive(&wq_empty[ws]);   // the group's last atom of the stage
      }
    }
    if (warp >= 8) goto done;   // the epilogue is one warpgroup (TMEM lane quarters 0-3)
    // Epilogue: TMEM lanes = tile rows, columns = tokens.
    if (!dead && !mbar_wait(acc_full, 0)) dead = true;
    dead = __any_sync(0xffffffffu, dead);   // TMEM loads are warp-collective
    tc_fence_after();
    const int q4 = warp - 4;                          // lane quarter
    const uint32_t trow = tmem + ((uint32_t)(32 * q4) << 16);
    float rs = 1.0f;
    if (FMT == FMT_INT8_ROW) {
      const int nrow = (MODE == TC_GATEUP) ? n0 + (r & 63) : n0 + r;
      const __half* rsp = (MODE == TC_GATEUP && r >= 64) ? job.rs1 : job.rs0;
      if (nrow < job.N) rs = __half2float(rsp[nrow]);
    }
    float* xch = reinterpret_cast<float*>(gbase + (a_base - base));   // A ring, free after the MMAs
    constexpr int CW = NT < 32 ? NT : 32;                              // columns per TMEM load
    for (int cc = 0; cc < NT; cc += CW) {
      float v[32];
      if (!dead) {
        if (CW == 32) {
          tmem_ld32(trow + cc, v);
        } else {
          uint32_t u[16];
          asm volatile(
              "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
              : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
                "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]),
                "=r"(u[15])
              : "r"(trow + cc));
          asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(u[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < CW; ++i) v[i] *= rs;
      if (MODE == TC_GATEUP) {
        if (r >= 64) {
#pragma unroll
          for (int i = 0; i < CW; ++i) xch[i * 64 + (r - 64)] = v[i];
        }
        named_sync(1, 128);
        if (r < 64 && !dead) {
          const int n = n0 + r;
          uint16_t* out = job.shared ? a.out_act_s : a.out_act;
#pragma unroll
          for (int i = 0; i < CW; ++i) {
            const int tok = cc + i;
            if (tok < tn && n < job.N)
              out[(size_t)(row_tok + tok) * job.N + n] = float_to_bf16_bits(gated_act(v[i], xch[i * 64 + r], a.act));
          }
        }
        named_sync(1, 128);
      } else if (!dead) {
        const int n = n0 + r;
        float* d = job.shared ? a.out_d_s : a.out_d;
        const int nslots = job.shared ? a.M : a.slots;
        if (n < job.N) {
#pragma unroll
          for (int i = 0; i < CW; ++i) {
            const int tok = cc + i;
            if (tok < tn) d[((size_t)split * nslots + row_tok + tok) * job.N + n] = v[i];
          }
        }
      }
    }
    tc_fence_before();
  }
done:
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, T::kTmemCols);
  }
}

template <int FMT, int NT, int MODE>
cudaError_t launch_t(const TcGemmArgs& a, dim3 grid, cudaStream_t s) {
  auto kern = k_qgemm_tc<FMT, NT, MODE>;
  constexpr size_t smem = tc_smem_bytes<FMT, NT>();
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  return launch_pdl(kern, grid, dim3(kThreads), smem, s, a);
}

template <int FMT, int MODE>
cudaError_t launch_nt(const TcGemmArgs& a, dim3 grid, cudaStream_t s) {
  switch (a.nt) {
    case 16: return launch_t<FMT, 16, MODE>(a, grid, s);
    case 32: return launch_t<FMT, 32, MODE>(a, grid, s);
    case 64: return launch_t<FMT, 64, MODE>(a, grid, s);
    case 128: return launch_t<FMT, 128, MODE>(a, grid, s);
    case 256: return launch_t<FMT, 256, MODE>(a, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

size_t tc_gemm_smem(int fmt, int nt) {
  const size_t stage = fmt == FMT_INT4_G32 ? TcFmt<FMT_INT4_G32>::kStageBytes : TcFmt<FMT_INT8_ROW>::kStageBytes;
  const int sb = nt >= 256 ? 3 : 4;
  const int sw = nt <= 128 ? 4 : 2;
  const int sa = nt <= 32 ? 8 : (nt <= 64 ? 6 : 4);
  return 2048 + sw * stage + (size_t)sa * kAtomBytes + (size_t)sb * nt * 128;
}

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

cudaError_t encode_tc_x_map(CUtensorMap* m, const uint16_t* x, int rows, int K, int nt) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, rows, (uint64_t)K * 2, 64, nt,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

cudaError_t launch_tc_gemm(const TcGemmArgs& a, int row_tiles, int splits, int jobs, cudaStream_t s) {
  const dim3 grid(row_tiles, a.token_tiles * splits, jobs);
  if (a.fmt == FMT_INT4_G32)
    return a.mode == TC_GATEUP ? launch_nt<FMT_INT4_G32, TC_GATEUP>(a, grid, s) : launch_nt<FMT_INT4_G32, TC_DOWN>(a, grid, s);
  return a.mode == TC_GATEUP ? launch_nt<FMT_INT8_ROW, TC_GATEUP>(a, grid, s) : launch_nt<FMT_INT8_ROW, TC_DOWN>(a, grid, s);
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
