// gelu.cu -- GELU (tanh form), bf16 -> bf16, fp32 arithmetic.
//
// Not part of the method on the pages: it joins the up- and down-projections
// of the DiT MLP workload (image-token-scale transformer block), so that the
// down-projection is fed what a real block feeds it.  HBM-bound, 4 bytes per
// element; 128-bit loads and stores of 8 elements, four of them in flight per
// thread before any is computed (one at a time left about 32 KB in flight per
// SM, too little to cover the DRAM latency).
#include <cuda_bf16.h>

#include "act.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace w8a8 {
namespace {

__device__ __forceinline__ uint32_t gelu2(uint32_t v) {
  float a, b;
  gelu_tanh_pair(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u), a, b);
  const __nv_bfloat162 r = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t *>(&r);
}

__global__ void gelu_kernel(const uint4 *__restrict__ x, uint4 *__restrict__ y, int64_t n8,
                            const uint16_t *__restrict__ xt, uint16_t *__restrict__ yt,
                            int64_t tail) {
  constexpr int kU = 4;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += kU * stride) {
    uint4 v[kU];
#pragma unroll
    for (int k = 0; k < kU; ++k)
      if (i + k * stride < n8) v[k] = ld_stream_u4(x + i + k * stride);
#pragma unroll
    for (int k = 0; k < kU; ++k)
      if (i + k * stride < n8)
        y[i + k * stride] = make_uint4(gelu2(v[k].x), gelu2(v[k].y), gelu2(v[k].z), gelu2(v[k].w));
  }
  if (blockIdx.x == 0 && threadIdx.x < tail) {
    const float a = gelu_tanh_f(__uint_as_float((uint32_t)xt[threadIdx.x] << 16));
    const __nv_bfloat16 r = __float2bfloat16_rn(a);
    yt[threadIdx.x] = *reinterpret_cast<const uint16_t *>(&r);
  }
}

}  // namespace
}  // namespace w8a8

using namespace w8a8;

extern "C" w8a8_status w8a8_gelu_tanh(const void *x, void *y, int64_t n, w8a8_stream_t stream) {
  if (!x || !y || n < 0) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return W8A8_ERR_ALIGNMENT;
  if (n == 0) return W8A8_OK;
  const int64_t n8 = n / 8, tail = n % 8;
  const int64_t blocks =
      std::max<int64_t>(1, std::min<int64_t>((n8 + 1023) / 1024, (int64_t)sm_count() * 8));
  gelu_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(x), static_cast<uint4 *>(y), n8,
      static_cast<const uint16_t *>(x) + n8 * 8, static_cast<uint16_t *>(y) + n8 * 8, tail);
  count_launch();
  return from_cuda(cudaGetLastError());
}
