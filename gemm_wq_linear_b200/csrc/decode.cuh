// In-register weight decode for the wq kernels (sm_100a).
//
// Each decoder turns packed 32-bit words into bf16 pairs (or fp32 values) with a
// few bit operations, in the spirit of the SIMT bit-parallel dequantization of
// the FP6-LLM / TC-FPx article (m.zhengruan.com news 124379, section
// "重新设计内核方案": dequantize inside registers with bit-level parallelism and
// splice the 2-bit and 4-bit pieces of each 6-bit weight in parallel).
//
// Pair convention: a decoded pair register holds (lo, hi) = (k, k + 1); the
// packers place the codes inside each word so that this needs no permutation.
#pragma once
#include <cstdint>

namespace wq {

// bf16 bit pattern of 128.0 in both halves: OR-ing a 4-bit code into the low
// mantissa bits gives the exact value 128 + q.
constexpr uint32_t kBf16Magic128x2 = 0x43004300u;

__device__ __forceinline__ uint32_t rotl32(uint32_t x, int s) { return __funnelshift_l(x, x, s); }

// int4: word w holds q[8t + 2r + h] in bits 4r + 16h .. +3.  Output p[r] = bf16
// pair (128 + q[8t + 2r], 128 + q[8t + 2r + 1]), r = 0..3.
__device__ __forceinline__ void decode_int4_word(uint32_t w, uint32_t p[4]) {
  p[0] = (w & 0x000F000Fu) | kBf16Magic128x2;
  p[1] = ((w >> 4) & 0x000F000Fu) | kBf16Magic128x2;
  p[2] = ((w >> 8) & 0x000F000Fu) | kBf16Magic128x2;
  p[3] = ((w >> 12) & 0x000F000Fu) | kBf16Magic128x2;
}

// FP6 (2+4 planes): p2 is the 2-bit-plane word of 16 weights, p4a / p4b the two
// 4-bit-plane words of its first and second 8 weights.  Output p[4c + j] = bf16
// pair (k = 8c + 2j, 8c + 2j + 1) holding code value * 2^-124 (subnormal for e = 0).
__device__ __forceinline__ void decode_fp6_words(uint32_t p2, uint32_t p4a, uint32_t p4b, uint32_t p[8]) {
  constexpr uint32_t kFour = 0x01E001E0u;  // bits 5..8 of each half: (e1 e0 m1 m0)
  constexpr uint32_t kTwo = 0x82008200u;   // bits 15 and 9 of each half: sign, e2
  p[0] = (p4a & kFour) | (p2 & kTwo);
  p[1] = (rotl32(p4a, 4) & kFour) | (rotl32(p2, 1) & kTwo);
  p[2] = (rotl32(p4a, 8) & kFour) | (rotl32(p2, 4) & kTwo);
  p[3] = (rotl32(p4a, 12) & kFour) | (rotl32(p2, 5) & kTwo);
  p[4] = (p4b & kFour) | (rotl32(p2, 8) & kTwo);
  p[5] = (rotl32(p4b, 4) & kFour) | (rotl32(p2, 9) & kTwo);
  p[6] = (rotl32(p4b, 8) & kFour) | (rotl32(p2, 12) & kTwo);
  p[7] = (rotl32(p4b, 12) & kFour) | (rotl32(p2, 13) & kTwo);
}

// int8 (offset binary): byte i of w is q + 128.  Output fp32 q for each byte:
// the byte is placed in the low mantissa of 2^23 (exact 2^23 + q + 128), then
// the constant is subtracted exactly.
__device__ __forceinline__ void decode_int8_word(uint32_t w, float v[4]) {
  constexpr float kBias = 8388608.0f + 128.0f;
  v[0] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540)) - kBias;
  v[1] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7541)) - kBias;
  v[2] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7542)) - kBias;
  v[3] = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7543)) - kBias;
}

// acc += a * b with a, b the low (or high) bf16 of a pair register; fp32
// accumulate, one rounding (mixed-precision FMA of sm_100).
__device__ __forceinline__ void fma_bf16_lo(float& acc, uint32_t a, uint32_t b) {
  asm("{.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, al, bl, %0;}\n"
      : "+f"(acc)
      : "r"(a), "r"(b));
}
__device__ __forceinline__ void fma_bf16_hi(float& acc, uint32_t a, uint32_t b) {
  asm("{.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %1;\n\t"
      "mov.b32 {bl, bh}, %2;\n\t"
      "fma.rn.f32.bf16 %0, ah, bh, %0;}\n"
      : "+f"(acc)
      : "r"(a), "r"(b));
}
// acc += a.lo * b.lo + a.hi * b.hi (two roundings, in that order).
__device__ __forceinline__ void fma_bf16x2(float& acc, uint32_t a, uint32_t b) {
  fma_bf16_lo(acc, a, b);
  fma_bf16_hi(acc, a, b);
}

// (acc0, acc1) += (w0 * x0, w1 * x1): packed fp32 FMA of sm_100 (one
// instruction for two lanes), each product rounded once into its accumulator.
__device__ __forceinline__ void ffma2(float& acc0, float& acc1, float w0, float w1, float x0, float x1) {
  asm("{.reg .b64 a, w, x;\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "mov.b64 w, {%2, %3};\n\t"
      "mov.b64 x, {%4, %5};\n\t"
      "fma.rn.f32x2 a, w, x, a;\n\t"
      "mov.b64 {%0, %1}, a;}\n"
      : "+f"(acc0), "+f"(acc1)
      : "f"(w0), "f"(w1), "f"(x0), "f"(x1));
}

// Exact bf16 pair -> two floats.
__device__ __forceinline__ float bf16_lo_f(uint32_t p) { return __uint_as_float(p << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t p) { return __uint_as_float(p & 0xFFFF0000u); }

// Pack two floats into a bf16 pair with round-to-nearest-even.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}


}  // namespace wq
