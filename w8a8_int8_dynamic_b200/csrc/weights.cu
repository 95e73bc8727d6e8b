// weights.cu -- load-time weight preparation beyond the plain repack:
//
// * online quantisation ("Online Quantization", Overview: quantised weights
//   and scales computed while the model loads; "Issue 5 probe: int8
//   quantized DiT serve paths on the RTX 3090", Round one: per-output-channel
//   symmetric): bf16 W[N, K] -> fp32 w_scale[N] and the packed int8 tile
//   image, in one kernel (one CTA per output channel);
// * compressed-tensors storage ("Issue 5 probe ...", Artifact: pack_to_int32,
//   four unsigned bytes of weight + 128 to a word): int32 words -> packed
//   int8 tiles.
//   Element 4j+i of a row is byte i (bits 8i..8i+7) of word j, stored as
//   w + 128, so in memory order the bytes are simply (w XOR 0x80): the plain
//   repack with each byte's top bit flipped.
//
// The per-channel rule is the activation rule of quant.cu: scale = amax/127
// (IEEE division), code = rint_half_even(w / scale), zero rows get scale 0.
#include "internal.h"
#include "ptx.cuh"

namespace w8a8 {
namespace {

__device__ __forceinline__ float lo_bf16(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ int code_of(float x, float s, float inv, bool exact_only) {
  if (exact_only) return __float2int_rn(__fdiv_rn(x, s));
  const float y = __fmul_rn(x, inv);
  const float r = rintf(y);
  if (fabsf(y - r) > 0.4999f) return __float2int_rn(__fdiv_rn(x, s));
  return (int)r;
}

__device__ __forceinline__ uint32_t bytes4(int a, int b, int c, int d) {
  const uint32_t ab = __byte_perm((uint32_t)a, (uint32_t)b, 0x0040);
  const uint32_t cd = __byte_perm((uint32_t)c, (uint32_t)d, 0x0040);
  return __byte_perm(ab, cd, 0x5410);
}

// One CTA per packed row n (n < Np).  Each thread owns 16-column chunks of
// the row (one packed 16-byte chunk each).  Pass 1: row amax; pass 2: codes
// written straight into the tile image (padding rows / columns -> zeros).
__global__ void __launch_bounds__(512) quant_pack_weight_kernel(
    const uint16_t *__restrict__ w, int N, int K, int kblocks, uint8_t *__restrict__ packed,
    float *__restrict__ w_scale) {
  const int n = blockIdx.x;
  const int nch = kblocks * 8;  // 16-byte chunks per packed row
  const bool real_row = n < N;
  const uint16_t *wr = w + (int64_t)(real_row ? n : 0) * K;
  uint32_t mx = 0;
  if (real_row) {
    for (int c = threadIdx.x; c < nch; c += blockDim.x) {
      const int k = c * 16;
      if (k < K) {
        const uint4 a = *reinterpret_cast<const uint4 *>(wr + k);
        const uint4 b = *reinterpret_cast<const uint4 *>(wr + k + 8);
        mx = __vmaxu2(mx, a.x & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, a.y & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, a.z & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, a.w & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, b.x & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, b.y & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, b.z & 0x7FFF7FFFu);
        mx = __vmaxu2(mx, b.w & 0x7FFF7FFFu);
      }
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
  const float s = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
  const float inv = amax == 0.0f ? 0.0f : __frcp_rn(s);
  const bool exact_only = s < 1e-30f;
  if (real_row && threadIdx.x == 0) w_scale[n] = s;

  const int nb = n >> 7, r = n & 127;
  for (int c = threadIdx.x; c < nch; c += blockDim.x) {
    const int kb = c >> 3, j = c & 7;  // k-block and logical 16-byte chunk in it
    const int k = c * 16;
    uint4 out = make_uint4(0, 0, 0, 0);
    if (real_row && amax != 0.0f && k < K) {
      const uint4 a = *reinterpret_cast<const uint4 *>(wr + k);
      const uint4 b = *reinterpret_cast<const uint4 *>(wr + k + 8);
      out.x = bytes4(code_of(lo_bf16(a.x), s, inv, exact_only), code_of(hi_bf16(a.x), s, inv, exact_only),
                     code_of(lo_bf16(a.y), s, inv, exact_only), code_of(hi_bf16(a.y), s, inv, exact_only));
      out.y = bytes4(code_of(lo_bf16(a.z), s, inv, exact_only), code_of(hi_bf16(a.z), s, inv, exact_only),
                     code_of(lo_bf16(a.w), s, inv, exact_only), code_of(hi_bf16(a.w), s, inv, exact_only));
      out.z = bytes4(code_of(lo_bf16(b.x), s, inv, exact_only), code_of(hi_bf16(b.x), s, inv, exact_only),
                     code_of(lo_bf16(b.y), s, inv, exact_only), code_of(hi_bf16(b.y), s, inv, exact_only));
      out.w = bytes4(code_of(lo_bf16(b.z), s, inv, exact_only), code_of(hi_bf16(b.z), s, inv, exact_only),
                     code_of(lo_bf16(b.w), s, inv, exact_only), code_of(hi_bf16(b.w), s, inv, exact_only));
    }
    const int64_t off = ((int64_t)nb * kblocks + kb) * 16384 + r * 128 + ((j ^ (r & 7)) << 4);
    *reinterpret_cast<uint4 *>(packed + off) = out;
  }
}

}  // namespace
}  // namespace w8a8

using namespace w8a8;

extern "C" w8a8_status w8a8_quant_pack_weight(const void *w, int64_t N, int64_t K, void *packed,
                                              size_t packed_bytes, float *w_scale,
                                              w8a8_stream_t stream) {
  if (!w || !packed || !w_scale) return W8A8_ERR_INVALID_ARG;
  if (N < 1 || K < 1) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0 || N > ((int64_t)1 << 30))
    return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(w) || !aligned16(packed) || !aligned16(w_scale)) return W8A8_ERR_ALIGNMENT;
  const int64_t need = packed_rows(N) * packed_cols(K);
  if ((int64_t)packed_bytes < need) return W8A8_ERR_BUFFER_TOO_SMALL;
  const int kblocks = (int)(packed_cols(K) / 128);
  const int nch = kblocks * 8;
  int threads = nch < 512 ? nch : 512;
  threads = (threads + 31) / 32 * 32;
  quant_pack_weight_kernel<<<(unsigned)packed_rows(N), (unsigned)threads, 0,
                             reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t *>(w), (int)N, (int)K, kblocks, static_cast<uint8_t *>(packed),
      w_scale);
  count_launch();
  return from_cuda(cudaGetLastError());
}
