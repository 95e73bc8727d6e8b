// act.cuh -- the activation that may follow a layer's dequantising epilogue.
//
// GELU (tanh form), the nonlinearity between the up- and down-projections of
// the DiT MLP workload (not part of the quantisation method on the pages).
// One definition serves the standalone kernel (gelu.cu) and the GEMM
// epilogues, with every fp32 step rounded explicitly, so the fused epilogue
// is bit-identical to "epilogue, then the standalone kernel".
#pragma once

#include <cuda_bf16.h>

#include "f32x2.cuh"
#include "w8a8.h"

namespace w8a8 {

// GELU_tanh(x) = 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3),
// evaluated as x * sigma(2u) (0.5 (1 + tanh(u)) = 1 / (1 + e^-2u)), with sigma
// written so nothing cancels: e = exp(-2|u|) in (0, 1], sigma = 1 / (1 + e)
// for u >= 0 and e / (1 + e) otherwise.  (1 + tanh(u) in fp32 is exactly 0
// once tanh(u) rounds to -1, which would flush small negative outputs to -0.)
// u has the sign of x, and 2|u| log2(e) = |x| (A + B x^2) with A = 2 sqrt(2/pi)
// log2(e) and B = 0.044715 A.
//
// Only the exponential uses the special-function unit (ex2.approx, which
// keeps subnormals: for x in about [-10.6, -10] the output is an fp32
// subnormal that bf16 still represents).  The reciprocal of d = 1 + e in
// (1, 2] is Newton-Raphson from the linear start 24/17 - 8/17 d (relative
// error at most 1/17 on [1, 2]; each step squares it: 2 steps, 1.2e-5), kept
// negated (s = -1/d) so each step is one FMA and one multiply.  Error budget,
// relative: the exponent argument carries <= 3 fp32 roundings on |t| <= 150
// (< 150 * 3 * 2^-24 absolute, < 2e-5 after the exponential); ex2.approx a
// few fp32 ulps; the reciprocal 1.2e-5; in all below 2^-14.5, far inside half
// a bf16 ulp (2^-9), so the bf16 result is the correctly rounded one except
// next to a rounding boundary (then 1 ulp away).
//
// Two values at a time: the arithmetic runs on sm_100's paired fp32
// instructions (fma/mul/add.rn.f32x2, each lane rounded exactly like the
// scalar instruction), which halves the instruction count of a kernel that
// is otherwise bound by instruction issue.  The one-value form runs the same
// pair code, so every caller gets the same bits.
__device__ __forceinline__ float ex2_approx(float t) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
}


__device__ __forceinline__ void gelu_tanh_pair(float x0, float x1, float &y0, float &y1) {
  const float A = 2.3022081981443250f;   // 2 sqrt(2/pi) log2(e)
  const float B = 0.10294323958002350f;  // 0.044715 A
  const uint64_t ax = f2_pack(fabsf(x0), fabsf(x1));
  const uint64_t nt = f2_mul(ax, f2_fma(f2_mul(ax, ax), f2_splat(-B), f2_splat(-A)));  // -t
  float nt0, nt1;
  f2_unpack(nt, nt0, nt1);
  const float e0 = ex2_approx(nt0), e1 = ex2_approx(nt1);  // exp(-2|u|)
  const uint64_t d = f2_add(f2_pack(e0, e1), f2_splat(1.0f));
  uint64_t s = f2_fma(d, f2_splat(0.47058823529411764f), f2_splat(-1.4117647058823530f));
#pragma unroll
  for (int i = 0; i < 2; ++i) s = f2_mul(s, f2_fma(d, s, f2_splat(2.0f)));  // s = -1/d
  const uint64_t n = f2_pack(signbit(x0) ? e0 : 1.0f, signbit(x1) ? e1 : 1.0f);
  f2_unpack(f2_mul(f2_mul(f2_pack(-x0, -x1), n), s), y0, y1);  // x n / d
}

__device__ __forceinline__ float gelu_tanh_f(float x) {
  float y, unused;
  gelu_tanh_pair(x, x, y, unused);
  return y;
}

__device__ __forceinline__ float round_bf16(float t) {
  return __bfloat162float(__float2bfloat16_rn(t));
}

// The epilogue's value t (before its final bf16 rounding) -> the value whose
// bf16 rounding is the layer output: t itself, or GELU of the rounded t.
__device__ __forceinline__ float apply_act(float t, int act) {
  return act == W8A8_ACT_GELU_TANH ? gelu_tanh_f(round_bf16(t)) : t;
}

// The same for two values at once.
__device__ __forceinline__ void apply_act_pair(float &t0, float &t1, int act) {
  if (act == W8A8_ACT_GELU_TANH) gelu_tanh_pair(round_bf16(t0), round_bf16(t1), t0, t1);
}

}  // namespace w8a8
