// quant.cu -- int8 activation quantisation, one symmetric scale per token
// computed at run time.
//
// Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
// Round two (the int8 activations of the W8A8 path, the scaled_int8_quant
// op); "Online Quantization", Parameters (activation_scheme "dynamic":
// scales computed at run time).
//
// Per row m:  amax = max_k |x[m,k]|;  s = amax / 127 (IEEE fp32 division);
//             q = clamp(rint_half_even(x / s), -127, 127);  amax == 0 -> s = 0, q = 0.
//
// Each row is handled by W warps (W = 1 for rows of up to 1024 elements,
// more for longer rows), each lane holding 4 16-byte chunks of the row in
// registers (8 when the input has enough rows that fewer, fatter warps pay;
// 16 for rows too long for 16 warps), all loaded at once with 128-bit
// streaming loads: the row is read exactly once and many loads are in
// flight per warp.  The row
// maximum is a packed 16-bit integer max on the bf16 magnitudes (|x| order
// equals the order of the 15 low bits for finite bf16), reduced with warp
// shuffles (and, for W > 1, one shared-memory step); each lane then writes
// its codes as 8-byte stores.  CTAs are small (about 128 threads: several
// rows per CTA when W = 1), so a GEMM CTA launched behind this kernel can
// share an SM with it.  Rows longer than 65536 elements take a two-pass
// kernel.  HBM-bound: 2 bytes read + 1 byte written per element.
//
// Both kernels are programmatic dependent launches: their CTAs may become
// resident while the preceding kernel of the stream is still running (the
// decode GEMM releases its dependents early), and wait on the device for it
// to complete before reading x, which may be that kernel's output.
//
// The per-element arithmetic (the code from one step of reciprocal
// refinement, rint by one addition) is in quant_common.cuh.

#include <cuda_bf16.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"
#include "quant_common.cuh"

namespace w8a8 {
namespace {

// W warps per row, R rows per CTA (blockDim = 32 * W * R), CPL chunks per
// lane.  Warp w of a row covers chunks [w * 32 * CPL, (w + 1) * 32 * CPL),
// lane l the chunks w * 32 * CPL + 32 j + l.  AHEAD: the instance launched
// ahead of a GEMM (same code; a function of its own, since the shared-memory
// carveout is a property of the function).
// zero_rows (nullable): a per-row word set to 0 here, before the GEMM behind
// this kernel folds its output maxima into it.
template <int CPL, bool AHEAD>
__global__ void __launch_bounds__(512) quant_warps_kernel(const uint16_t *__restrict__ x,
                                                          int64_t ldx, int M, int K, int W, int R,
                                                          int8_t *__restrict__ q,
                                                          float *__restrict__ a_scale,
                                                          uint32_t *__restrict__ zero_rows) {
  // Let a dependent GEMM start its prologue while the rows are quantised.
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rl = warp / W, w = warp - rl * W;
  const int64_t row = (int64_t)blockIdx.x * R + rl;
  const bool row_ok = row < M;
  if (zero_rows && row_ok && w == 0 && lane == 0) zero_rows[row] = 0u;
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
  for (int j = 0; j < CPL; ++j) mx = absmax_chunk(mx, v[j]);
  uint32_t m = absmax_fold(mx);
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
  uint2 out[CPL];
  if (s >= 1e-30f) {
    if constexpr (CPL >= 8) {
      // Long rows keep the issue slots busy (close to instruction-bound):
      // there the paired fp32 instructions take two instructions an element
      // off (4096 x 12288: 25.4-25.9 -> 25.0-25.5 us alone, 2048 x 12288:
      // 14.5 -> 14.1 us, on one box).  Short rows wait on DRAM latency, and
      // there the pair form measured no faster or slower.
      const uint64_t ns2 = f2_splat(-s), inv2 = f2_splat(inv), rnd2 = f2_splat(kRound);
#pragma unroll
      for (int j = 0; j < CPL; ++j) out[j] = codes8_x2(v[j], ns2, inv2, rnd2);
    } else {
#pragma unroll
      for (int j = 0; j < CPL; ++j) out[j] = codes8(v[j], s, inv);
    }
  } else {
#pragma unroll
    for (int j = 0; j < CPL; ++j) out[j] = codes8_ieee(v[j], s);
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
    float *__restrict__ a_scale, uint32_t *__restrict__ zero_rows) {
  griddep_launch_dependents();
  griddep_wait();  // x may be the preceding kernel's output
  const int64_t row = blockIdx.x;
  if (zero_rows && threadIdx.x == 0) zero_rows[row] = 0u;
  const int nchunks = K >> 3;
  const uint16_t *xr = x + row * ldx;
  uint32_t mx = 0;
  for (int i = threadIdx.x; i < nchunks; i += blockDim.x) {
    const uint4 c = *reinterpret_cast<const uint4 *>(xr + (int64_t)i * 8);
    mx = absmax_chunk(mx, c);
  }
  uint32_t m = absmax_fold(mx);
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
      out = exact_only ? codes8_ieee(c, s) : codes8(c, s, inv);
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
      out.x = pack4((uint32_t)quant_static_one(bf16_lo(a.x), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(a.x), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_lo(a.y), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(a.y), s, inv, exact_only));
      out.y = pack4((uint32_t)quant_static_one(bf16_lo(a.z), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(a.z), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_lo(a.w), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(a.w), s, inv, exact_only));
      out.z = pack4((uint32_t)quant_static_one(bf16_lo(b.x), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(b.x), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_lo(b.y), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(b.y), s, inv, exact_only));
      out.w = pack4((uint32_t)quant_static_one(bf16_lo(b.z), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(b.z), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_lo(b.w), s, inv, exact_only),
                    (uint32_t)quant_static_one(bf16_hi(b.w), s, inv, exact_only));
    }
    *reinterpret_cast<uint4 *>(q + m * K + k) = out;
  }
}

// Ahead of a GEMM, every SM that runs quantisation blocks is set up for the
// largest shared-memory share.  The GEMM launched behind them needs about
// 214 KB of shared memory a CTA; an SM configured for a small share (the
// default for a kernel that uses 64 bytes) takes such a CTA only after it has
// drained, so the GEMM would start no earlier than the quantisation ends.
// Alone, the quantisation keeps the default share: with the largest one (and
// so the smallest L1) a 512 x 4096 input takes 4.5 us instead of 3.9 us.
FuncAttrOnce g_carveout[8];  // one per kernel instance (`slot`)

template <typename Kernel>
void prefer_max_shared(Kernel k, int slot) {
  if (g_carveout[slot].ensure([&] {
        return cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    (int)cudaSharedmemCarveoutMaxShared);
      }) != cudaSuccess)
    (void)cudaGetLastError();  // a preference only: the launch goes ahead without it
}

// Launches k, as a programmatic dependent of the preceding kernel of the
// stream when `pdl`.  `slot` >= 0 names k for the one-time carveout setting
// (kernels launched ahead of a GEMM); -1 leaves the default.
template <typename... Params, typename... Args>
cudaError_t launch_dependent(void (*k)(Params...), int slot, bool pdl, dim3 grid, dim3 block,
                             cudaStream_t stream, Args... args) {
  if (slot >= 0) prefer_max_shared(k, slot);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, static_cast<Params>(args)...);
}

}  // namespace

w8a8_status launch_quant(const void *x, int64_t M, int64_t K, int64_t ldx, int8_t *q,
                         float *a_scale, cudaStream_t stream, bool ahead_of_gemm,
                         uint32_t *zero_rows) {
  const int64_t nchunks = K / 8;
  const uint16_t *xp = static_cast<const uint16_t *>(x);
  // Chunks per lane (a power of two): 4 where the row has that many per lane;
  // 8 when the M x W warps of the launch would exceed about two waves of
  // resident warps (SMs x 112): fewer, fatter warps then keep more loads in
  // flight per thread (4096 x 12288 rows: 25.6 us against 28.6 us with 4);
  // 16 only where a row would need more than 16 warps.  Fewer than 4 would
  // quantise a few rows faster alone (512 x 4096: 3.4 us with 1 chunk per
  // lane against 4.2 us), but its bigger CTAs leave a GEMM CTA no room
  // beside them, and the layer step loses more than that (16.9 -> 17.4 us).
  const int64_t per_lane = (nchunks + 31) / 32;
  const int64_t warp_budget = (int64_t)sm_count() * 112;
  int cpl = 1;
  while (cpl < 4 && cpl < per_lane) cpl *= 2;
  while (cpl < 16 && cpl < per_lane) {
    const int64_t w = (nchunks + 32 * cpl - 1) / (32 * cpl);
    if (w > 16 || (cpl < 8 && M * w > warp_budget))
      cpl *= 2;
    else
      break;
  }
  const int64_t W = (nchunks + 32 * cpl - 1) / (32 * cpl);
  // Inside a layer the quantisation is a programmatic dependent of the
  // preceding kernel (after the small-M kernel, which releases its
  // dependents early, it becomes resident and waits on the device).  Alone,
  // an input resident in one wave (at most 16 warps a SM on average) is a
  // plain launch: launches of it back to back, each released at the start of
  // the one before, would sit resident and waiting on the slots the running
  // launch needs (512 x 4096: 3.96 -> 3.08 us).  Longer inputs are
  // dependents there too: the next launch's first CTAs then start as the
  // running one's last wave drains (4096 x 3072: 11.3 -> 10.7 us; 4096 x
  // 12288: 32.3 -> 31.3 us).
  const bool pdl = ahead_of_gemm || M * W > (int64_t)sm_count() * 16;
  cudaError_t e = cudaSuccess;
  if (W > 16) {
    // 1024-thread CTAs never leave room for a GEMM CTA: default carveout.
    e = launch_dependent(quant_rows_two_pass_kernel, -1, pdl, dim3((unsigned)M), dim3(1024),
                         stream, xp, ldx, (int)K, q, a_scale, zero_rows);
  } else {
    const int R = W >= 4 ? 1 : (int)(4 / W);  // rows per CTA: about 128 threads
    const unsigned grid = (unsigned)((M + R - 1) / R);
    const unsigned threads = (unsigned)(32 * W * R);
    // The instance with the largest carveout where the GEMM behind it can
    // start beside it: every CTA resident at once, at most 16 warps a SM on
    // average (the 512-row layers).  Longer inputs run in several waves, in
    // which the GEMM could start only during the last; they keep the default
    // carveout and its larger L1.
    const bool wide = ahead_of_gemm && M * W <= (int64_t)sm_count() * 16;
    switch (cpl) {
#define W8A8_QUANT_CASE(C, SLOT)                                                          \
  case C:                                                                                 \
    e = wide ? launch_dependent(quant_warps_kernel<C, true>, SLOT, pdl, dim3(grid),       \
                                dim3(threads), stream, xp, ldx, (int)M, (int)K,           \
                                (int)W, R, q, a_scale, zero_rows)                         \
             : launch_dependent(quant_warps_kernel<C, false>, -1, pdl, dim3(grid),        \
                                dim3(threads), stream, xp, ldx, (int)M, (int)K,           \
                                (int)W, R, q, a_scale, zero_rows);                        \
    break;
      W8A8_QUANT_CASE(1, 0)
      W8A8_QUANT_CASE(2, 1)
      W8A8_QUANT_CASE(4, 2)
      W8A8_QUANT_CASE(8, 3)
      W8A8_QUANT_CASE(16, 4)
#undef W8A8_QUANT_CASE
      default:
        return W8A8_ERR_INVALID_ARG;
    }
  }
  if (e != cudaSuccess) return from_cuda(e);
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
  return launch_quant(x, M, K, ldx, q, a_scale, reinterpret_cast<cudaStream_t>(stream), false,
                      nullptr);
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
