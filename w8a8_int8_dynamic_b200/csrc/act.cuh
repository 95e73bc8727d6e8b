// act.cuh -- the activation that may follow a layer's dequantising epilogue.
//
// GELU (tanh form), the nonlinearity between the up- and down-projections of
// the DiT MLP workload (not part of the quantisation method on the pages).
// One definition serves the standalone kernel (gelu.cu) and the GEMM
// epilogues, with every fp32 step rounded explicitly, so the fused epilogue
// is bit-identical to "epilogue, then the standalone kernel".
#pragma once

#include <cuda_bf16.h>

#include "w8a8.h"

namespace w8a8 {

// GELU_tanh(x) = 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3),
// evaluated as x * sigma(2u) (0.5 (1 + tanh(u)) = 1 / (1 + e^-2u)), with sigma
// written so nothing cancels: e = exp(-2|u|) in (0, 1], sigma = 1 / (1 + e)
// for u >= 0 and e / (1 + e) otherwise.  (1 + tanh(u) in fp32 is exactly 0
// once tanh(u) rounds to -1, which would flush small negative outputs to -0.)
//
// exp and the reciprocal are the hardware approximations (ex2.approx and
// rcp.approx, both keeping subnormals: for x in about [-10.6, -10] the output
// is an fp32 subnormal that bf16 still represents).  Error budget, relative:
// u and the exponent argument carry <= 4 fp32 roundings on |2u log2 e| <= 150,
// i.e. < 150 * 4 * 2^-24 absolute in the exponent -> < 2.5e-5 after exp;
// ex2.approx and rcp.approx add a few fp32 ulps; the total stays below 2^-15,
// far inside half a bf16 ulp (2^-9), so the bf16 result is the correctly
// rounded one except next to a rounding boundary (then 1 ulp away).
__device__ __forceinline__ float ex2_approx(float t) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
}

__device__ __forceinline__ float rcp_approx(float t) {
  float r;
  asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(t));
  return r;
}

__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float c = 0.7978845608028654f;  // sqrt(2 / pi)
  const float x3 = __fmul_rn(__fmul_rn(x, x), x);
  const float u = __fmul_rn(c, __fadd_rn(x, __fmul_rn(0.044715f, x3)));
  const float e = ex2_approx(__fmul_rn(-2.8853900817779268f, fabsf(u)));  // exp(-2|u|)
  const float sig = __fmul_rn(u >= 0.0f ? 1.0f : e, rcp_approx(__fadd_rn(1.0f, e)));
  return __fmul_rn(x, sig);
}

__device__ __forceinline__ float round_bf16(float t) {
  return __bfloat162float(__float2bfloat16_rn(t));
}

// The epilogue's value t (before its final bf16 rounding) -> the value whose
// bf16 rounding is the layer output: t itself, or GELU of the rounded t.
__device__ __forceinline__ float apply_act(float t, int act) {
  return act == W8A8_ACT_GELU_TANH ? gelu_tanh_f(round_bf16(t)) : t;
}

}  // namespace w8a8
