// quant_common.cuh -- the per-element arithmetic of the activation
// quantisation ("Issue 5 probe: int8 quantized DiT serve paths on the RTX
// 3090", Round two: int8 activations, one symmetric scale per token computed
// at run time), used by the quantisation kernels (quant.cu).
//
// Per row: amax = max |x|, s = RN(amax / 127), code = rint_half_even(RN(x / s)).
//
// The code without a division.  The quotient is formed from inv = RN(1/s) by
// reciprocal refinement (P. W. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1),
// 1990): q0 = RN(x inv), r0 = x - s q0 (exact, one FMA), q1 = RN(q0 + r0 inv).
// In general q1 is within an ulp of x / s but not always RN(x / s) -- a
// second step would make it so (Markstein's Theorem 1) -- yet only rint(q1)
// matters here, and rint(q1) = rint(RN(x / s)) for every bf16 x with |x| <=
// amax and s = RN(amax / 127) >= 1e-30: all 523,084,815 such (amax, x >= 0)
// pairs were checked (the operations are odd in x, so negative x follow).
// Without the step, 5296 of them differ.  So: one multiply and two FMAs per
// element, no branch.  Smaller scales (1/s no longer finite and normal) take
// the IEEE quotient.  |x| <= amax makes |x / s| <= 127 (1 + 2^-23), so no
// clamp is needed.
//
// rint without a conversion: for |y| < 2^22, RN(y + 1.5 * 2^23) is
// 1.5 * 2^23 + rint(y) (round-half-even, the unit in the last place being 1
// there), so the low byte of its bit pattern is the two's-complement code.
#pragma once

#include <stdint.h>

#include "f32x2.cuh"

namespace w8a8 {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Running maximum of the bf16 magnitudes of one 16-byte chunk, as two packed
// 16-bit lanes (for finite bf16, |x| order is the order of the 15 low bits).
__device__ __forceinline__ uint32_t absmax_chunk(uint32_t m, const uint4 &v) {
  m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
  return __vmaxu2(m, v.w & 0x7FFF7FFFu);
}

// The two packed lanes of absmax_chunk -> one magnitude's bit pattern.
__device__ __forceinline__ uint32_t absmax_fold(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

// A quotient whose nearest integer is that of RN(x / s), from inv = RN(1/s)
// (one refinement step, see above; for codes only).
__device__ __forceinline__ float code_quotient(float x, float s, float inv) {
  const float q0 = __fmul_rn(x, inv);
  const float r0 = __fmaf_rn(-s, q0, x);
  return __fmaf_rn(r0, inv, q0);
}

// Low bytes of four ints -> one word.
__device__ __forceinline__ uint32_t pack4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t ab = __byte_perm(a, b, 0x0040);
  const uint32_t cd = __byte_perm(c, d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

constexpr float kRound = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ uint32_t code_bits(float x, float s, float inv) {
  return __float_as_uint(__fadd_rn(code_quotient(x, s, inv), kRound));
}

// One 16-byte chunk (8 bf16) -> its 8 codes, for s >= 1e-30.
__device__ __forceinline__ uint2 codes8(const uint4 &v, float s, float inv) {
  return make_uint2(pack4(code_bits(bf16_lo(v.x), s, inv), code_bits(bf16_hi(v.x), s, inv),
                          code_bits(bf16_lo(v.y), s, inv), code_bits(bf16_hi(v.y), s, inv)),
                    pack4(code_bits(bf16_lo(v.z), s, inv), code_bits(bf16_hi(v.z), s, inv),
                          code_bits(bf16_lo(v.w), s, inv), code_bits(bf16_hi(v.w), s, inv)));
}

// The same two values at a time on the paired fp32 instructions (each lane
// rounded like the scalar ones, so the codes are the same bits): the bf16
// pair of one 32-bit word, ns2 = (-s, -s), inv2 = (inv, inv), rnd2 =
// (kRound, kRound).  Half the floating-point instructions of codes8.
__device__ __forceinline__ void code_bits_x2(uint32_t w, uint64_t ns2, uint64_t inv2,
                                             uint64_t rnd2, uint32_t &lo, uint32_t &hi) {
  const uint64_t x = f2_pack(bf16_lo(w), bf16_hi(w));
  const uint64_t q0 = f2_mul(x, inv2);
  const uint64_t r0 = f2_fma(ns2, q0, x);
  float b0, b1;
  f2_unpack(f2_add(f2_fma(r0, inv2, q0), rnd2), b0, b1);
  lo = __float_as_uint(b0);
  hi = __float_as_uint(b1);
}

__device__ __forceinline__ uint2 codes8_x2(const uint4 &v, uint64_t ns2, uint64_t inv2,
                                           uint64_t rnd2) {
  uint32_t c[8];
  code_bits_x2(v.x, ns2, inv2, rnd2, c[0], c[1]);
  code_bits_x2(v.y, ns2, inv2, rnd2, c[2], c[3]);
  code_bits_x2(v.z, ns2, inv2, rnd2, c[4], c[5]);
  code_bits_x2(v.w, ns2, inv2, rnd2, c[6], c[7]);
  return make_uint2(pack4(c[0], c[1], c[2], c[3]), pack4(c[4], c[5], c[6], c[7]));
}

// The same with the IEEE quotient (rows with s < 1e-30).  A rolled loop keeps
// a single copy of the division code.
__device__ __forceinline__ uint2 codes8_ieee(const uint4 &v, float s) {
  uint32_t o0 = 0, o1 = 0;
#pragma unroll 1
  for (int h = 0; h < 8; ++h) {
    const uint32_t word = h < 2 ? v.x : h < 4 ? v.y : h < 6 ? v.z : v.w;
    const float xv = (h & 1) ? bf16_hi(word) : bf16_lo(word);
    const uint32_t code = (uint32_t)__float2int_rn(__fdiv_rn(xv, s)) & 0xFFu;
    if (h < 4)
      o0 |= code << ((h & 3) * 8);
    else
      o1 |= code << ((h & 3) * 8);
  }
  return make_uint2(o0, o1);
}

}  // namespace w8a8
