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
// One CTA per row.  The row is read once with 128-bit streaming loads and
// held in registers (1, 2 or 4 16-byte chunks per thread for rows of up to
// 8192 / 16384 / 32768 elements; longer rows take a two-pass kernel); the row
// maximum is a packed 16-bit integer max on the bf16 magnitudes (|x| order
// equals the order of the 15 low bits for finite bf16), reduced with warp
// shuffles and one shared-memory step; each thread then writes its codes as
// packed 8-byte stores.  HBM-bound: 2 bytes read + 1 byte written per element.
//
// Exact quotient at reciprocal speed: the code of x is rint(RN(x / s)).
// With inv = RN(1/s), y = RN(x * inv) is within 3 * 2^-24 * 127 < 2.3e-5 of
// RN(x / s) (|x / s| <= 127 + tiny).  So when y is farther than 1e-4 from a
// half-integer, rint(y) == rint(RN(x / s)); otherwise (rarely) the kernel
// computes the IEEE quotient itself with __fdiv_rn.  Rows with s < 1e-30
// (where 1/s could overflow) always take the IEEE quotient.
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
__device__ __forceinline__ int quant_one(float x, float s, float inv, bool exact_only) {
  if (exact_only) return __float2int_rn(__fdiv_rn(x, s));
  const float y = __fmul_rn(x, inv);
  const float r = rintf(y);
  if (fabsf(y - r) > 0.4999f) return __float2int_rn(__fdiv_rn(x, s));
  return (int)r;
}

// Low bytes of four ints -> one word (byte permutes).
__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d) {
  const uint32_t ab = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);
  const uint32_t cd = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

template <int CHUNKS>
__global__ void __launch_bounds__(1024) quant_rows_kernel(const uint16_t *__restrict__ x,
                                                          int64_t ldx, int K,
                                                          int8_t *__restrict__ q,
                                                          float *__restrict__ a_scale) {
  // Let a dependent GEMM start its prologue while the rows are quantised.
  griddep_launch_dependents();

  const int64_t row = blockIdx.x;
  const int nchunks = K >> 3;  // 8 bf16 per 16-byte chunk
  const uint16_t *xr = x + row * ldx;
  uint4 v[CHUNKS];
  uint32_t mx = 0;  // packed pair of 16-bit magnitudes
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    const int i = threadIdx.x + j * blockDim.x;
    if (i < nchunks) {
      v[j] = ld_stream_u4(xr + (int64_t)i * 8);
      mx = __vmaxu2(mx, v[j].x & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, v[j].y & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, v[j].z & 0x7FFF7FFFu);
      mx = __vmaxu2(mx, v[j].w & 0x7FFF7FFFu);
    } else {
      v[j] = make_uint4(0, 0, 0, 0);
    }
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
  if (amax == 0.0f) {
    if (threadIdx.x == 0) a_scale[row] = 0.0f;
#pragma unroll
    for (int j = 0; j < CHUNKS; ++j) {
      const int i = threadIdx.x + j * blockDim.x;
      if (i < nchunks) *reinterpret_cast<uint2 *>(qr + (int64_t)i * 8) = make_uint2(0, 0);
    }
    return;
  }
  const float s = __fdiv_rn(amax, 127.0f);
  const float inv = __frcp_rn(s);
  const bool exact_only = s < 1e-30f;
  if (threadIdx.x == 0) a_scale[row] = s;
#pragma unroll
  for (int j = 0; j < CHUNKS; ++j) {
    const int i = threadIdx.x + j * blockDim.x;
    if (i < nchunks) {
      const uint4 c = v[j];
      const uint32_t lo = pack4(quant_one(bf16_lo(c.x), s, inv, exact_only),
                                quant_one(bf16_hi(c.x), s, inv, exact_only),
                                quant_one(bf16_lo(c.y), s, inv, exact_only),
                                quant_one(bf16_hi(c.y), s, inv, exact_only));
      const uint32_t hi = pack4(quant_one(bf16_lo(c.z), s, inv, exact_only),
                                quant_one(bf16_hi(c.z), s, inv, exact_only),
                                quant_one(bf16_lo(c.w), s, inv, exact_only),
                                quant_one(bf16_hi(c.w), s, inv, exact_only));
      *reinterpret_cast<uint2 *>(qr + (int64_t)i * 8) = make_uint2(lo, hi);
    }
  }
}

// Rows longer than 32768 elements: two passes over the row (the second one
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
  // One CTA per row with as many threads as the row has 16-byte chunks (up
  // to 1024): the row is read in one wave of loads and each warp has little
  // serial work, which is what this latency-bound kernel needs.
  const int64_t nchunks = K / 8;
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  auto threads_for = [&](int per) {
    int64_t t = (nchunks + per - 1) / per;
    return round_up(t < 32 ? 32 : t, 32);
  };
  // at most 512 threads per row-CTA (measured: 768-thread CTAs fit only two
  // per SM and run the 12288-wide rows slower than 384-thread ones)
  if (threads_for(1) <= 512) {
    quant_rows_kernel<1><<<(unsigned)M, (unsigned)threads_for(1), 0, stream>>>(xp, ldx, (int)K, q,
                                                                                 a_scale);
  } else if (threads_for(2) <= 512) {
    quant_rows_kernel<2><<<(unsigned)M, (unsigned)threads_for(2), 0, stream>>>(xp, ldx, (int)K, q,
                                                                                 a_scale);
  } else if (threads_for(4) <= 1024) {
    quant_rows_kernel<4><<<(unsigned)M, (unsigned)threads_for(4), 0, stream>>>(xp, ldx, (int)K, q,
                                                                                 a_scale);
  } else {
    quant_rows_two_pass_kernel<<<(unsigned)M, 1024, 0, stream>>>(xp, ldx, (int)K, q, a_scale);
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
