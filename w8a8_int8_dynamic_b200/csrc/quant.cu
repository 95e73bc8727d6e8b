// quant.cu -- dynamic per-token symmetric int8 activation quantisation.
//
// Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
// Round two ("dynamic per-token symmetric int8 activations", the
// scaled_int8_quant op); "Online Quantization", Parameters
// (activation_scheme "dynamic": scales computed at run time).
//
// Per row m:  amax = max_k |x[m,k]|;  s = amax / 127 (IEEE fp32 division);
//             q = clamp(rint_half_even(x / s), -127, 127);  amax == 0 -> s = 0, q = 0.
//
// Each row is handled by W warps (W = 1 for rows of up to 1024 elements,
// more for longer rows), each lane holding up to 4 16-byte chunks of the row
// in registers (8 or 16 for rows longer than 16384), all loaded at once with
// 128-bit streaming loads: the row is read exactly once and many loads are in
// flight per warp.  The row
// maximum is a packed 16-bit integer max on the bf16 magnitudes (|x| order
// equals the order of the 15 low bits for finite bf16), reduced with warp
// shuffles (and, for W > 1, one shared-memory step); each lane then writes
// its codes as 8-byte stores.  CTAs are small (about 128 threads: several
// rows per CTA when W = 1), so a GEMM CTA launched behind this kernel can
// share an SM with it.  Rows longer than 65536 elements take a two-pass
// kernel.  HBM-bound: 2 bytes read + 1 byte written per element.
//
// Exact quotient without a division: the code of x is rint(RN(x / s)).
// RN(x / s) is formed from inv = RN(1/s) by reciprocal refinement (P. W.
// Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990, Theorem 1: if y is 1/b rounded to
// nearest and q is within one ulp of a/b, then r = a - b q is exact and
// RN(q + r y) = RN(a/b)).  q0 = RN(x inv) is within 1.5 ulp of x / s, so one
// refinement step first brings it within one ulp (q1 = RN(q0 + r0 inv) with
// r0 = RN(x - s q0): |q1 - x/s| <= ulp/2 + 1.5 ulp * 2^-24), and a second
// step, Markstein's, gives RN(x / s) exactly: 1 multiply + 4 FMAs per
// element, no branch.  rint is then one addition (see kRound).  Rows with
// s < 1e-30 (where 1/s could overflow) take the IEEE quotient.  |x| <= amax
// makes |x / s| <= 127 (1 + 2^-23), so no clamp is needed.
#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace w8a8 {
namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Code of one element: rint(RN(x / s)).  y = RN(x * inv) is within 2.3e-5 of
// RN(x / s), so rint(y) is the answer unless y lies within 1e-4 of a
// half-integer, i.e. |y - rint(y)| > 0.4999 (it is always <= 0.5); only then
// is the IEEE quotient formed.  |x| <= amax makes |y| <= 127 (1 + 2^-22), so
// the result is always in [-127, 127] and needs no clamp.
// The IEEE quotient path, out of line: it runs rarely, and inlined at every
// element of an unrolled row it would bloat the kernel past the instruction
// cache.
static __device__ __noinline__ int exact_code(float x, float s) {
  return __float2int_rn(__fdiv_rn(x, s));
}

__device__ __forceinline__ int quant_one(float x, float s, float inv, bool exact_only) {
  if (exact_only) return exact_code(x, s);
  const float y = __fmul_rn(x, inv);
  const float r = rintf(y);
  if (fabsf(y - r) > 0.49997f) return exact_code(x, s);
  return (int)r;
}

// Low bytes of four ints -> one word (byte permutes).
// RN(x / s) from inv = RN(1/s) (Markstein refinement, see above).
__device__ __forceinline__ float quotient_rn(float x, float s, float inv) {
  const float q0 = __fmul_rn(x, inv);
  const float r0 = __fmaf_rn(-s, q0, x);
  const float q1 = __fmaf_rn(r0, inv, q0);
  const float r1 = __fmaf_rn(-s, q1, x);
  return __fmaf_rn(r1, inv, q1);
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  const uint32_t ab = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);
  const uint32_t cd = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// W warps per row, R rows per CTA (blockDim = 32 * W * R), CPL chunks per
// lane.  Warp w of a row covers chunks [w * 32 * CPL, (w + 1) * 32 * CPL),
// lane l the chunks w * 32 * CPL + 32 j + l.
template <int CPL>
__global__ void __launch_bounds__(512) quant_warps_kernel(const uint16_t *__restrict__ x,
                                                          int64_t ldx, int M, int K, int W, int R,
                                                          int8_t *__restrict__ q,
                                                          float *__restrict__ a_scale) {
  // Let a dependent GEMM start its prologue while the rows are quantised.
  griddep_launch_dependents();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rl = warp / W, w = warp - rl * W;
  const int64_t row = (int64_t)blockIdx.x * R + rl;
  const bool row_ok = row < M;
  const int nchunks = K >> 3;  // 8 bf16 per 16-byte chunk
  const int c0 = w * 32 * CPL + lane;
  const uint16_t *xr = x + (row_ok ? row : 0) * ldx;
  // All loads first (so they are in flight together), then the maximum.
  uint4 v[CPL];
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = c0 + 32 * j;
    v[j] = make_uint4(0, 0, 0, 0);
    if (row_ok && c < nchunks) v[j] = ld_stream_u4(xr + (int64_t)c * 8);
  }
  uint32_t mx = 0;  // packed pair of 16-bit magnitudes
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    mx = __vmaxu2(mx, v[j].x & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v[j].y & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v[j].z & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, v[j].w & 0x7FFF7FFFu);
  }
  uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (W > 1) {
    __shared__ uint32_t warp_max[16];
    if (lane == 0) warp_max[warp] = m;
    __syncthreads();
    for (int i = 0; i < W; ++i) m = max(m, warp_max[rl * W + i]);
  }
  if (!row_ok) return;

  const float amax = __uint_as_float(m << 16);
  int8_t *qr = q + row * (int64_t)K;
  if (amax == 0.0f) {
    if (w == 0 && lane == 0) a_scale[row] = 0.0f;
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const int c = c0 + 32 * j;
      if (c < nchunks) *reinterpret_cast<uint2 *>(qr + (int64_t)c * 8) = make_uint2(0, 0);
    }
    return;
  }
  const float s = __fdiv_rn(amax, 127.0f);
  const float inv = __frcp_rn(s);
  if (w == 0 && lane == 0) a_scale[row] = s;
  // Rounding: for |y| < 2^22, RN(y + 1.5 * 2^23) is 1.5 * 2^23 + rint(y)
  // (round-half-even: the unit in the last place is 1 there), so its low
  // byte is the two's-complement code: no conversion instruction needed.
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  uint2 out[CPL];
  if (s >= 1e-30f) {
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      const uint32_t e[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      uint32_t code[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        code[2 * h] = __float_as_uint(__fadd_rn(quotient_rn(bf16_lo(e[h]), s, inv), kRound));
        code[2 * h + 1] = __float_as_uint(__fadd_rn(quotient_rn(bf16_hi(e[h]), s, inv), kRound));
      }
      out[j] = make_uint2(pack4((int)code[0], (int)code[1], (int)code[2], (int)code[3]),
                          pack4((int)code[4], (int)code[5], (int)code[6], (int)code[7]));
    }
  } else {
    // subnormal-scale rows: the IEEE quotient (rolled: a single copy of the
    // division code)
#pragma unroll
    for (int j = 0; j < CPL; ++j) {
      uint32_t o0 = 0, o1 = 0;
#pragma unroll 1
      for (int h = 0; h < 8; ++h) {
        const uint32_t word = h < 2 ? v[j].x : h < 4 ? v[j].y : h < 6 ? v[j].z : v[j].w;
        const float xv = (h & 1) ? bf16_hi(word) : bf16_lo(word);
        const uint32_t code = (uint32_t)__float2int_rn(__fdiv_rn(xv, s)) & 0xFFu;
        const int sh = (h & 3) * 8;
        if (h < 4)
          o0 |= code << sh;
        else
          o1 |= code << sh;
      }
      out[j] = make_uint2(o0, o1);
    }
  }
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = c0 + 32 * j;
    if (c < nchunks) *reinterpret_cast<uint2 *>(qr + (int64_t)c * 8) = out[j];
  }
}

// Rows longer than 65536 elements: two passes over the row (the second one
// hits L2), same arithmetic.
__global__ void __launch_bounds__(1024) quant_rows_two_pass_kernel(
    const uint16_t *__restrict__ x, int64_t ldx, int K, int8_t *__restrict__ q,
    float *__restrict__ a_scale) {
  griddep_launch_dependents();
  const int64_t row = blockIdx.x;
  const int nchunks = K >> 3;
  const uint16_t *xr = x + row * ldx;
  uint32_t mx = 0;
  for (int i = threadIdx.x; i < nchunks; i += blockDim.x) {
    const uint4 c = *reinterpret_cast<const uint4 *>(xr + (int64_t)i * 8);
    mx = __vmaxu2(mx, c.x & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, c.y & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, c.z & 0x7FFF7FFFu);
    mx = __vmaxu2(mx, c.w & 0x7FFF7FFFu);
  }
  uint32_t m = max(mx & 0xFFFFu, mx >> 16);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t warp_max[32];
  __shared__ uint32_t row_max;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) warp_max[warp] = m;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    uint32_t t = lane < nw ? warp_max[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t = max(t, __shfl_xor_sync(0xFFFFFFFFu, t, o));
    if (lane == 0) row_max = t;
  }
  __syncthreads();
  const float amax = __uint_as_float(row_max << 16);
  int8_t *qr = q + row * (int64_t)K;
  const float s = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
  const float inv = amax == 0.0f ? 0.0f : __frcp_rn(s);
  const bool exact_only = s < 1e-30f;
  if (threadIdx.x == 0) a_scale[row] = s;
  for (int i = threadIdx.x; i < nchunks; i += blockDim.x) {
    uint2 out = make_uint2(0, 0);
    if (amax != 0.0f) {
      const uint4 c = *reinterpret_cast<const uint4 *>(xr + (int64_t)i * 8);
      out.x = pack4(quant_one(bf16_lo(c.x), s, inv, exact_only),
                    quant_one(bf16_hi(c.x), s, inv, exact_only),
                    quant_one(bf16_lo(c.y), s, inv, exact_only),
                    quant_one(bf16_hi(c.y), s, inv, exact_only));
      out.y = pack4(quant_one(bf16_lo(c.z), s, inv, exact_only),
                    quant_one(bf16_hi(c.z), s, inv, exact_only),
                    quant_one(bf16_lo(c.w), s, inv, exact_only),
                    quant_one(bf16_hi(c.w), s, inv, exact_only));
    }
    *reinterpret_cast<uint2 *>(qr + (int64_t)i * 8) = out;
  }
}

// Static (calibrated) per-tensor scale: code = clamp(rint(RN(x / scale)),
// -127, 127); a scale that is not > 0 gives codes 0 and a_scale 0.  The scale
// is read from device memory, so a calibrated value can change without a host
// round trip.  One thread per 16-element chunk (32 bytes in, 16 bytes out),
// grid-stride over all M * K/16 chunks.  The reciprocal shortcut holds while
// |y| <= 256 (error < 256 * 3 * 2^-24 < 1e-4 of the quotient); beyond that
// the code saturates either way.  Scales outside [1e-30, 1e30] (where RN(1/s)
// overflows or goes subnormal) always take the IEEE quotient.
__device__ __forceinline__ int quant_static_one(float x, float s, float inv, bool exact_only) {
  float v;
  if (exact_only) {
    v = rintf(__fdiv_rn(x, s));
  } else {
    const float y = __fmul_rn(x, inv);
    if (fabsf(y) > 256.0f) return y > 0.0f ? 127 : -127;
    v = rintf(y);
    if (fabsf(y - v) > 0.4999f) v = rintf(__fdiv_rn(x, s));
  }
  v = fminf(fmaxf(v, -127.0f), 127.0f);
  return (int)v;
}

__global__ void __launch_bounds__(256) quant_static_kernel(const uint16_t *__restrict__ x,
                                                           int64_t ldx, int64_t M, int K,
                                                           const float *__restrict__ scale_ptr,
                                                           int8_t *__restrict__ q,
                                                           float *__restrict__ a_scale) {
  griddep_launch_dependents();
  const float s_in = *scale_ptr;
  const bool usable = s_in > 0.0f;  // false for NaN
  const float s = usable ? s_in : 0.0f;
  const bool exact_only = !(s >= 1e-30f && s <= 1e30f);
  const float inv = exact_only ? 0.0f : __frcp_rn(s);
  const int per_row = K >> 4;
  const int64_t total = M * per_row;
  for (int64_t c = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; c < total;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t m = c / per_row;
    const int k = (int)(c - m * per_row) * 16;
    if (k == 0 && a_scale) a_scale[m] = s;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (usable) {
      const uint16_t *src = x + m * ldx + k;
      const uint4 a = ld_stream_u4(src);
      const uint4 b = ld_stream_u4(src + 8);
      out.x = pack4(quant_static_one(bf16_lo(a.x), s, inv, exact_only),
                    quant_static_one(bf16_hi(a.x), s, inv, exact_only),
                    quant_static_one(bf16_lo(a.y), s, inv, exact_only),
                    quant_static_one(bf16_hi(a.y), s, inv, exact_only));
      out.y = pack4(quant_static_one(bf16_lo(a.z), s, inv, exact_only),
                    quant_static_one(bf16_hi(a.z), s, inv, exact_only),
                    quant_static_one(bf16_lo(a.w), s, inv, exact_only),
                    quant_static_one(bf16_hi(a.w), s, inv, exact_only));
      out.z = pack4(quant_static_one(bf16_lo(b.x), s, inv, exact_only),
                    quant_static_one(bf16_hi(b.x), s, inv, exact_only),
                    quant_static_one(bf16_lo(b.y), s, inv, exact_only),
                    quant_static_one(bf16_hi(b.y), s, inv, exact_only));
      out.w = pack4(quant_static_one(bf16_lo(b.z), s, inv, exact_only),
                    quant_static_one(bf16_hi(b.z), s, inv, exact_only),
                    quant_static_one(bf16_lo(b.w), s, inv, exact_only),
                    quant_static_one(bf16_hi(b.w), s, inv, exact_only));
    }
    *reinterpret_cast<uint4 *>(q + m * K + k) = out;
  }
}

}  // namespace

w8a8_status launch_quant(const void *x, int64_t M, int64_t K, int64_t ldx, int8_t *q,
                         float *a_scale, cudaStream_t stream) {
  const int64_t nchunks = K / 8;
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  // Chunks per lane: the smallest power of two covering the row with one
  // warp, at most 4 (measured: 4 chunks per lane and more warps per row beat
  // 16 per lane on every shape), more only where the row would need more than
  // 16 warps; then warps per row.
  const int64_t per_lane = (nchunks + 31) / 32;
  int cpl = 1;
  while (cpl < per_lane && (cpl < 4 || (nchunks + 32 * cpl - 1) / (32 * cpl) > 16) && cpl < 16)
    cpl *= 2;
  const int64_t W = (nchunks + 32 * cpl - 1) / (32 * cpl);
  if (W > 16) {
    quant_rows_two_pass_kernel<<<(unsigned)M, 1024, 0, stream>>>(xp, ldx, (int)K, q, a_scale);
  } else {
    const int R = W >= 4 ? 1 : (int)(4 / W);  // rows per CTA: about 128 threads
    const unsigned grid = (unsigned)((M + R - 1) / R);
    const unsigned threads = (unsigned)(32 * W * R);
    switch (cpl) {
#define W8A8_QUANT_CASE(C)                                                                     \
  case C:                                                                                      \
    quant_warps_kernel<C><<<grid, threads, 0, stream>>>(xp, ldx, (int)M, (int)K, (int)W, R, q, \
                                                        a_scale);                              \
    break;
      W8A8_QUANT_CASE(1)
      W8A8_QUANT_CASE(2)
      W8A8_QUANT_CASE(4)
      W8A8_QUANT_CASE(8)
      W8A8_QUANT_CASE(16)
#undef W8A8_QUANT_CASE
      default:
        return W8A8_ERR_INVALID_ARG;
    }
  }
  count_launch();
  return from_cuda(cudaGetLastError());
}

}  // namespace w8a8

using namespace w8a8;

extern "C" w8a8_status w8a8_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx,
                                      int8_t *q, float *a_scale, w8a8_stream_t stream) {
  if (!x || !q || !a_scale) return W8A8_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7FFFFFFF || K < 1 || ldx < K) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(q) || !aligned16(a_scale) || ldx % 8 != 0)
    return W8A8_ERR_ALIGNMENT;
  return launch_quant(x, M, K, ldx, q, a_scale, reinterpret_cast<cudaStream_t>(stream));
}


extern "C" w8a8_status w8a8_quant_act_static(const void *x, int64_t M, int64_t K, int64_t ldx,
                                             const float *scale, int8_t *q, float *a_scale,
                                             w8a8_stream_t stream) {
  if (!x || !q || !scale) return W8A8_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7FFFFFFF || K < 1 || ldx < K) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK) return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(x) || !aligned16(q) || ldx % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(scale) & 3u) || (a_scale && !aligned16(a_scale)))
    return W8A8_ERR_ALIGNMENT;
  const int64_t chunks = M * (K / 16);
  const int64_t blocks = std::min<int64_t>((chunks + 255) / 256, (int64_t)sm_count() * 8);
  quant_static_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t *>(x), ldx, M, (int)K, scale, q, a_scale);
  count_launch();
  return from_cuda(cudaGetLastError());
}
