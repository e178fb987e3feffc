// Arithmetic of the weight-streaming GEMV (gemv_tma.cu): activations staged as int16 fixed point per weight chunk,
// codes times staged activations summed exactly in int32 with DP2A.
#pragma once
#include "common.cuh"
#include "norm.cuh"

namespace moeffn {

// Activations are staged per weight chunk as int16 fixed point with one
// power-of-two factor per chunk: x = xi * 2^(e-14), e = floor(log2(max|x|)).
// A bf16 value has 8 significant bits, so every value within 2^7 of the
// chunk's largest is exact and the rest lose only bits below 2^(e-15).
// Codes times xi are then summed exactly in int32 with DP2A (two 16x8-bit
// products per instruction) and scaled once per chunk.
__device__ __forceinline__ int dp2a_lo_u(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_u(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_lo_s(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi_s(int a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

template <int FMT>
struct Codes;

// INT4: a chunk is one group of 32 codes (4 words). Word codes q0..q7: the
// low nibbles of its bytes are q0,q2,q4,q6 and the high nibbles q1,q3,q5,q7,
// so the staged int16 of a word are ordered x0,x2,x4,x6,x1,x3,x5,x7.
template <>
struct Codes<FMT_INT4_G32> {
  static constexpr int kChunk = 32;
  static constexpr int kStageBytes = 80;  // 64 bytes of int16 + 16 bytes pad (bank spread)
  static __device__ __forceinline__ int slot_of(int j) {  // position of element j of a word
    return (j & 1) * 4 + (j >> 1);
  }
  // Adds the 8 products of word w with its staged activations (16 bytes).
  static __device__ __forceinline__ void dot_word(uint32_t w, uint4 x, int& p0, int& p1) {
    const uint32_t lo = w & 0x0F0F0F0Fu, hi = (w >> 4) & 0x0F0F0F0Fu;
    p0 = dp2a_lo_u((int)x.x, lo, p0);
    p1 = dp2a_hi_u((int)x.y, lo, p1);
    p0 = dp2a_lo_u((int)x.z, hi, p0);
    p1 = dp2a_hi_u((int)x.w, hi, p1);
  }
};

// INT8: a chunk is 16 signed codes (4 words); staged in natural order.
template <>
struct Codes<FMT_INT8_ROW> {
  static constexpr int kChunk = 16;
  static constexpr int kStageBytes = 48;  // 32 bytes of int16 + 16 bytes pad
  static __device__ __forceinline__ int slot_of(int j) { return j; }
  // Two words (8 codes) with their staged activations (16 bytes).
  static __device__ __forceinline__ void dot_word(uint32_t w0, uint32_t w1, uint4 x, int& p0, int& p1) {
    p0 = dp2a_lo_s((int)x.x, w0, p0);
    p1 = dp2a_hi_s((int)x.y, w0, p1);
    p0 = dp2a_lo_s((int)x.z, w1, p0);
    p1 = dp2a_hi_s((int)x.w, w1, p1);
  }
};

// Q4_K: a chunk is one 32-weight sub-block, staged in natural order. A code
// run of 32 bytes holds two sub-blocks (low nibbles: weights 4w..4w+3 of
// word w of the first, high nibbles: of the second), so each nibble half of a
// word meets four consecutive staged values.
template <>
struct Codes<FMT_Q4K> {
  static constexpr int kChunk = 32;
  static constexpr int kStageBytes = 80;  // 64 bytes of int16 + 16 bytes pad
  static __device__ __forceinline__ int slot_of(int j) { return j; }
  // Words w0, w1 (codes 8h..8h+7 of both sub-blocks) with the staged values
  // 8h..8h+7 of the low (xl) and high (xh) sub-block.
  static __device__ __forceinline__ void dot_words(uint32_t w0, uint32_t w1, uint4 xl, uint4 xh, int& pl, int& ph) {
    const uint32_t l0 = w0 & 0x0F0F0F0Fu, h0 = (w0 >> 4) & 0x0F0F0F0Fu;
    const uint32_t l1 = w1 & 0x0F0F0F0Fu, h1 = (w1 >> 4) & 0x0F0F0F0Fu;
    pl = dp2a_lo_u((int)xl.x, l0, pl);
    pl = dp2a_hi_u((int)xl.y, l0, pl);
    pl = dp2a_lo_u((int)xl.z, l1, pl);
    pl = dp2a_hi_u((int)xl.w, l1, pl);
    ph = dp2a_lo_u((int)xh.x, h0, ph);
    ph = dp2a_hi_u((int)xh.y, h0, ph);
    ph = dp2a_lo_u((int)xh.z, h1, ph);
    ph = dp2a_hi_u((int)xh.w, h1, ph);
  }
};

// Stages one chunk of a bf16 activation row (p: the chunk's first element,
// 16-byte aligned; null for a zero pad row): the int16 values in code order
// at dst, the chunk's power-of-two factor in *xf and (INT4, Q4_K) its plain
// sum in *xsum, the sum the min term of the affine formats multiplies. With `wn`
// (the same chunk of an RMSNorm weight) the chunk is first normalized:
// x -> bf16(x * inv_rms * w).
template <int FMT>
__device__ __forceinline__ void stage_chunk(const uint16_t* p, uint8_t* dst, float* xf, float* xsum,
                                            const uint16_t* wn = nullptr, float inv_rms = 0.f) {
  using C = Codes<FMT>;
  uint16_t v[C::kChunk];
  if (p != nullptr) {
#pragma unroll
    for (int q = 0; q < C::kChunk / 8; ++q) {
      const uint4 u = __ldcg(reinterpret_cast<const uint4*>(p) + q);   // L2: rows other CTAs may have written
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        v[8 * q + 2 * j] = (uint16_t)(w[j] & 0xFFFFu);
        v[8 * q + 2 * j + 1] = (uint16_t)(w[j] >> 16);
      }
    }
    if (wn != nullptr) {
#pragma unroll
      for (int q = 0; q < C::kChunk / 8; ++q) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(wn) + q);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          v[8 * q + 2 * j] = prenorm_elem(v[8 * q + 2 * j], (uint16_t)(w[j] & 0xFFFFu), inv_rms);
          v[8 * q + 2 * j + 1] = prenorm_elem(v[8 * q + 2 * j + 1], (uint16_t)(w[j] >> 16), inv_rms);
        }
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < C::kChunk; ++j) v[j] = 0;
  }
  float amax = 0.f, sum = 0.f;
#pragma unroll
  for (int j = 0; j < C::kChunk; ++j) {
    const float f = bf16_bits_to_float(v[j]);
    amax = fmaxf(amax, fabsf(f));
    sum += f;
  }
  int16_t* d = reinterpret_cast<int16_t*>(dst);
  constexpr int kW = (C::kChunk == 32 ? 8 : 4);   // codes per 32-bit word
  // e = floor(log2(amax)) from the exponent field; the factors 2^(14-e) and
  // 2^(e-14) are then normal floats built from their exponent fields, and the
  // scaling is an exact multiplication. Chunks whose largest value is below
  // 2^-100 take the library path.
  const int eb = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
  if (amax > 0.f && eb >= -100) {
    const float up = __uint_as_float((uint32_t)(127 + 14 - eb) << 23);
#pragma unroll
    for (int j = 0; j < C::kChunk; ++j)
      d[(j / kW) * kW + C::slot_of(j % kW)] = (int16_t)__float2int_rn(bf16_bits_to_float(v[j]) * up);
    *xf = __uint_as_float((uint32_t)(127 + eb - 14) << 23);
  } else {
    int e = 0;
    if (amax > 0.f) {
      frexpf(amax, &e);
      e -= 1;                                   // amax in [2^e, 2^(e+1))
    }
#pragma unroll
    for (int j = 0; j < C::kChunk; ++j) {
      const float f = bf16_bits_to_float(v[j]);
      d[(j / kW) * kW + C::slot_of(j % kW)] = (int16_t)(amax > 0.f ? __float2int_rn(ldexpf(f, 14 - e)) : 0);
    }
    *xf = amax > 0.f ? ldexpf(1.0f, e - 14) : 0.f;
  }
  if (FMT == FMT_INT4_G32 || FMT == FMT_Q4K) *xsum = sum;
}

// Exact int32 dot products of one chunk of codes (wv: 16 bytes) with the
// chunk's staged activations at x (16-byte aligned): p0 + p1.
template <int FMT>
__device__ __forceinline__ int chunk_dot(uint4 wv, const uint8_t* x) {
  int p0 = 0, p1 = 0;
  if (FMT == FMT_INT4_G32) {
    const uint32_t w[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 x4 = *reinterpret_cast<const uint4*>(x + q * 16);
      Codes<FMT_INT4_G32>::dot_word(w[q], x4, p0, p1);
    }
  } else {
    const uint4 x0 = *reinterpret_cast<const uint4*>(x);
    const uint4 x1 = *reinterpret_cast<const uint4*>(x + 16);
    Codes<FMT_INT8_ROW>::dot_word(wv.x, wv.y, x0, p0, p1);
    Codes<FMT_INT8_ROW>::dot_word(wv.z, wv.w, x1, p0, p1);
  }
  return p0 + p1;
}

}  // namespace moeffn
