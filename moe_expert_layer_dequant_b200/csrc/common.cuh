// Shared device helpers of the quantized FFN / MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moeffn {

// Weight formats (values match moeffn_qformat in include/moeffn.h).
enum : int { FMT_INT8_ROW = 1, FMT_INT4_G32 = 2, FMT_BF16 = 3, FMT_F32 = 4, FMT_Q4K = 5 };
enum : int { ACT_SILU = 0, ACT_GELU_TANH = 1 };

// Device view of one quantized matrix W[N][K] (row-major, K contiguous).
//  INT8-row : q = int8 [N][K], scale = fp16 [N], mn = null.
//  INT4-g32 : q = uint8 [N][K/2] (element 2j = low nibble of byte j),
//             scale = fp16 [N][K/32], mn = fp16 [N][K/32]; w = q*scale + mn.
//  Q4_K     : q = [N][K/256] super-blocks of 144 bytes, scale = mn = null
//             (see Q4K below).
struct QW {
  const uint8_t* q;
  const __half* scale;
  const __half* mn;
};

// fp32 whose bit pattern is 2^23: OR-ing an integer below 2^23 into the
// mantissa gives the float 2^23 + integer exactly (the "magic number" int->float
// conversion used by fast dequantizers, e.g. Kim et al. 2022, "Who Says
// Elephants Can't Run", and FasterTransformer's int4 converters).
constexpr uint32_t kMagic = 0x4B000000u;
constexpr float kMagicF = 8388608.0f;  // 2^23

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t*>(&h);
}

__device__ __forceinline__ float round_bf16(float f) {
  return __bfloat162float(__float2bfloat16_rn(f));
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + expf(-g)); }

__device__ __forceinline__ float gelu_tanh_f(float g) {
  const float k0 = 0.7978845608028654f;  // sqrt(2/pi)
  return 0.5f * g * (1.0f + tanhf(k0 * (g + 0.044715f * g * g * g)));
}

__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }

__device__ __forceinline__ float gated_act(float g, float u, int act) {
  return (act == ACT_SILU ? silu_f(g) : gelu_tanh_f(g)) * u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16-byte streaming load of weight bytes: read once, so keep it out of L1.
__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ----------------------------------------------------------------------------
// Dequantized dot products of one 16-byte weight chunk with staged activations.
//
// Activations are staged in shared memory as fp32, pre-multiplied per element
// position by the power of two that undoes the position of the code inside
// its 32-bit word (so a code can be turned into a float with one LOP3 and no
// shift). Both scalings are exact.
// ----------------------------------------------------------------------------

// INT4: a 16-byte chunk is one group of 32 codes. Position i (0..7) of a word
// becomes q * 16^(i%4); the staged activation carries 16^-(i%4).
__device__ __forceinline__ float int4_pos_scale(int k) {
  const int i = (k & 7) & 3;
  return i == 0 ? 1.0f : (i == 1 ? 0.0625f : (i == 2 ? 0.00390625f : 0.000244140625f));
}

// INT8: a 16-byte chunk is 16 codes. Position i (0..3) of a word becomes
// q * 256^(i%2); the staged activation carries 256^-(i%2).
__device__ __forceinline__ float int8_pos_scale(int k) {
  return (k & 1) ? 0.00390625f : 1.0f;
}

// Codes of one word as positioned floats, minus the magic: q_i * 16^(i%4).
__device__ __forceinline__ void int4_word_codes(uint32_t w, float2 (&c)[4]) {
  const uint32_t hi = w >> 16;
  float2 a, b, d, e;
  a.x = __uint_as_float((w & 0x000Fu) | kMagic);
  a.y = __uint_as_float((w & 0x00F0u) | kMagic);
  b.x = __uint_as_float((w & 0x0F00u) | kMagic);
  b.y = __uint_as_float((w & 0xF000u) | kMagic);
  d.x = __uint_as_float((hi & 0x000Fu) | kMagic);
  d.y = __uint_as_float((hi & 0x00F0u) | kMagic);
  e.x = __uint_as_float((hi & 0x0F00u) | kMagic);
  e.y = __uint_as_float((hi & 0xF000u) | kMagic);
  const float2 m = make_float2(-kMagicF, -kMagicF);
  c[0] = __fadd2_rn(a, m);
  c[1] = __fadd2_rn(b, m);
  c[2] = __fadd2_rn(d, m);
  c[3] = __fadd2_rn(e, m);
}

// Signed int8 codes of one word: (byte ^ 0x80) = q + 128 is OR-ed into the
// mantissa, then 2^23 + 128 * 256^(i%2) is subtracted: q_i * 256^(i%2).
__device__ __forceinline__ void int8_word_codes(uint32_t w, float2 (&c)[2]) {
  const uint32_t hi = w >> 16;
  float2 a, b;
  a.x = __uint_as_float((w & 0x00FFu) ^ (0x0080u | kMagic));
  a.y = __uint_as_float((w & 0xFF00u) ^ (0x8000u | kMagic));
  b.x = __uint_as_float((hi & 0x00FFu) ^ (0x0080u | kMagic));
  b.y = __uint_as_float((hi & 0xFF00u) ^ (0x8000u | kMagic));
  const float2 m = make_float2(-(kMagicF + 128.0f), -(kMagicF + 32768.0f));
  c[0] = __fadd2_rn(a, m);
  c[1] = __fadd2_rn(b, m);
}

}  // namespace moeffn

namespace moeffn {

// Exact fp32 weights of the 8 INT4 codes of one word: q * s + m with q made by
// the magic-number conversion. q * s needs at most 4 + 11 significant bits and
// both terms are multiples of 2^-24, so the single rounding of fmaf is exact
// whenever |w| < 1 (and far beyond for the stated value ranges).
__device__ __forceinline__ void int4_word_dequant(uint32_t w, float s, float m, float (&out)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float q = __uint_as_float(((w >> (4 * i)) & 0xFu) | kMagic) - kMagicF;
    out[i] = fmaf(q, s, m);
  }
}

// Exact fp32 weights of the 4 signed INT8 codes of one word: q * s.
__device__ __forceinline__ void int8_word_dequant(uint32_t w, float s, float (&out)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float q = __uint_as_float(((w >> (8 * i)) & 0xFFu) ^ (0x80u | kMagic)) - (kMagicF + 128.0f);
    out[i] = q * s;
  }
}

// Q4_K super-block (the GGUF K-quant layout): 256 weights in 144 bytes,
//  bytes 0-1 d (fp16), 2-3 dmin (fp16), 4-15 the packed 6-bit scale and min
//  of sub-blocks 0..7 (32 weights each), 16-143 codes in four runs of 32
//  bytes: run c holds weights 64c..64c+31 in its low nibbles and
//  64c+32..64c+63 in its high nibbles. w = d * scale_j * q - dmin * min_j;
//  d * scale_j and dmin * min_j are exact in fp32, so fmaf(q, d * scale_j,
//  -dmin * min_j) is the exact value rounded once.
struct Q4K {
  static constexpr int kBlock = 256;
  static constexpr int kBytes = 144;
  // hdr: the block's first 16 bytes as four words (d | dmin << 16, then the
  // 12 packed bytes s[0..11]). Sub-blocks 0..3: scale = s[j] & 63, min =
  // s[j + 4] & 63; 4..7: low 4 bits from the nibbles of s[j + 4], top 2 bits
  // from the top of s[j - 4] (scale) and s[j] (min).
  static __device__ __forceinline__ void scale_min(const uint4& hdr, int j, float& sc, float& mn) {
    const uint32_t lo = hdr.y, mid = hdr.z, hi = hdr.w;   // s[0..3], s[4..7], s[8..11]
    uint32_t a, b;
    if (j < 4) {
      a = (lo >> (8 * j)) & 63u;
      b = (mid >> (8 * j)) & 63u;
    } else {
      const int i = j - 4;
      const uint32_t h = (hi >> (8 * i)) & 0xFFu;
      a = (h & 15u) | (((lo >> (8 * i + 6)) & 3u) << 4);
      b = (h >> 4) | (((mid >> (8 * i + 6)) & 3u) << 4);
    }
    const float d = __half2float(__ushort_as_half((unsigned short)(hdr.x & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half((unsigned short)(hdr.x >> 16)));
    sc = d * (float)a;
    mn = -(dmin * (float)b);
  }
};

}  // namespace moeffn

namespace moeffn {

// Programmatic dependent launch: a kernel launched with the PDL attribute may
// start while its predecessor in the stream still runs. It must call
// pdl_wait() before touching memory the predecessor writes or reads; weights
// (never written by kernels) may be streamed before that.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

}  // namespace moeffn
