// gemm_common.cuh -- pieces shared by the 1-SM and 2-SM GEMM kernels: tile
// constants, kernel arguments, and the dequantising epilogue (TMEM -> fp32 in
// the oracle's operation order -> bf16), which follows "Issue 5 probe: int8
// quantized DiT serve paths on the RTX 3090", Round two: per-token and
// per-output-channel fp32 scales on the int8 product, bf16 out.
#pragma once

#include <cuda_bf16.h>

#include "act.cuh"
#include "internal.h"
#include "ptx.cuh"

namespace w8a8 {

constexpr int kBM = 128;                 // tile rows (MMA M)
constexpr int kBK = 128;                 // bytes of K per pipeline stage
constexpr int kTileBytes = 128 * kBK;    // one 128 x 128 int8 tile = 16 KB
constexpr int kThreads = 192;            // 6 warps
constexpr int kDecodeNT = 16;            // activation rows per decode MMA (N)

struct GemmArgs {
  const uint8_t *packed_w;
  const float *a_scale;
  const float *w_scale;
  const uint16_t *bias;  // may be null
  void *out;             // bf16 [M, N] or int32 [M, N]
  int M, N;
  int num_kb;            // K blocks of 128 bytes (= packed K / 128)
  int tiles_m, tiles_n;
  int act;               // w8a8_act applied after the dequantisation
  int *status;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&r);
}

__device__ __forceinline__ float dequant(int32_t acc, float as, float ws) {
  return __fmul_rn(__fmul_rn(__int2float_rn(acc), as), ws);
}


// Stages this tile's per-column scale and bias into the warp's own smem
// slice (all lanes then read them as broadcasts).
template <int BN>
__device__ __forceinline__ void stage_columns(const GemmArgs &a, int nb, int lane, float *s_ws,
                                              uint16_t *s_bias) {
  const int n0 = nb * BN;
#pragma unroll
  for (int j = lane * 4; j < BN; j += 128) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n0 + j < a.N) v = __ldg(reinterpret_cast<const float4 *>(a.w_scale + n0 + j));
    *reinterpret_cast<float4 *>(s_ws + j) = v;
  }
  if (a.bias) {
#pragma unroll
    for (int j = lane * 8; j < BN; j += 256) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n0 + j < a.N) v = __ldg(reinterpret_cast<const uint4 *>(a.bias + n0 + j));
      *reinterpret_cast<uint4 *>(s_bias + j) = v;
    }
  }
}

// Drains one BN-column accumulator from TMEM: 32 columns per tcgen05.ld, the
// fp32 scale/bias arithmetic in the defined order, 16-byte bf16 stores.
template <int BN, bool OUT_I32>
__device__ __forceinline__ void epilogue_tile(const GemmArgs &a, uint32_t tmem_cols, int quarter,
                                              int lane, int row_base, int nb, float as,
                                              const float *s_ws, const uint16_t *s_bias) {
  // TMEM lane (quarter * 32 + lane) holds output row row_base + that lane
  const int row = row_base + quarter * 32 + lane;
  const bool row_ok = row < a.M;
  const uint32_t taddr = tmem_cols + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    const int n0 = nb * BN + c * 32;
    if (n0 >= a.N) break;  // uniform across the warp
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr + c * 32, r);
    tmem_ld_wait();
    if (OUT_I32) {
      if (row_ok) {
        int32_t *dst = static_cast<int32_t *>(a.out) + (int64_t)row * a.N + n0;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (n0 + 4 * g < a.N)
            *reinterpret_cast<uint4 *>(dst + 4 * g) =
                make_uint4(r[4 * g], r[4 * g + 1], r[4 * g + 2], r[4 * g + 3]);
      }
    } else {
      const float *ws = s_ws + c * 32;
      const uint16_t *bs = s_bias + c * 32;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int nn = n0 + 8 * g;
        if (nn >= a.N) break;  // N % 8 == 0: groups of 8 are all in or all out
        const float4 w0 = *reinterpret_cast<const float4 *>(ws + 8 * g);
        const float4 w1 = *reinterpret_cast<const float4 *>(ws + 8 * g + 4);
        float t[8];
        t[0] = dequant((int32_t)r[8 * g + 0], as, w0.x);
        t[1] = dequant((int32_t)r[8 * g + 1], as, w0.y);
        t[2] = dequant((int32_t)r[8 * g + 2], as, w0.z);
        t[3] = dequant((int32_t)r[8 * g + 3], as, w0.w);
        t[4] = dequant((int32_t)r[8 * g + 4], as, w1.x);
        t[5] = dequant((int32_t)r[8 * g + 5], as, w1.y);
        t[6] = dequant((int32_t)r[8 * g + 6], as, w1.z);
        t[7] = dequant((int32_t)r[8 * g + 7], as, w1.w);
        if (a.bias) {
          const uint4 b = *reinterpret_cast<const uint4 *>(bs + 8 * g);
          const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            t[2 * h] = __fadd_rn(t[2 * h], __uint_as_float(bw[h] << 16));
            t[2 * h + 1] = __fadd_rn(t[2 * h + 1], __uint_as_float(bw[h] & 0xFFFF0000u));
          }
        }
        if (a.act != W8A8_ACT_NONE) {
#pragma unroll
          for (int h = 0; h < 8; ++h) t[h] = apply_act(t[h], a.act);
        }
        if (row_ok) {
          uint16_t *dst = static_cast<uint16_t *>(a.out) + (int64_t)row * a.N + nn;
          *reinterpret_cast<uint4 *>(dst) =
              make_uint4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]),
                         pack_bf16x2(t[4], t[5]), pack_bf16x2(t[6], t[7]));
        }
      }
    }
  }
}


// Output staging for the TMA-store epilogue: each epilogue warp owns two
// 2 KB buffers, each a 32-row x 32-column bf16 box in the 64-byte-swizzle
// layout of the output tensor map (16-byte chunk c of row r at chunk position
// c ^ ((r >> 1) & 3)), so the 32 lanes' 16-byte writes spread over all banks.
constexpr int kEpiStageBytes = 32 * 32 * 2;
constexpr int kEpiStagePerWarp = 2 * kEpiStageBytes;

__device__ __forceinline__ uint32_t swz64_offset(int r, int c16) {
  return (uint32_t)(r * 64 + ((c16 ^ ((r >> 1) & 3)) << 4));
}

// Drains one BN-column accumulator from TMEM and writes it as bf16 through
// shared memory with one TMA store per 32 x 32 box (rows and columns outside
// the output are clipped by the tensor map).  `stage` is this warp's 4 KB.
// `extra`, when non-null, is an int32 partial in shared memory added to the
// accumulator before the scales (element (r, j) at extra_index(r, j)).
template <int BN, typename ExtraIndex>
__device__ __forceinline__ void epilogue_tile_tma(const GemmArgs &a, const CUtensorMap *tmap_y,
                                                  uint32_t tmem_cols, int quarter, int lane,
                                                  int row_base, int nb, float as,
                                                  const float *s_ws, const uint16_t *s_bias,
                                                  uint8_t *stage, uint32_t &stage_count,
                                                  const int32_t *extra, ExtraIndex extra_index) {
  const uint32_t taddr = tmem_cols + ((uint32_t)(quarter * 32) << 16);
  const int r = quarter * 32 + lane;  // row within the CTA's 128
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    const int n0 = nb * BN + c * 32;
    if (n0 >= a.N) break;  // uniform across the warp
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + c * 32, v);
    tmem_ld_wait();
    if (extra) {
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const uint4 p = *reinterpret_cast<const uint4 *>(extra + extra_index(r, c * 32 + 4 * g));
        v[4 * g] += p.x;
        v[4 * g + 1] += p.y;
        v[4 * g + 2] += p.z;
        v[4 * g + 3] += p.w;
      }
    }
    // the buffer written now was last used two boxes ago: its store must have
    // finished reading shared memory
    uint8_t *buf = stage + (stage_count & 1) * kEpiStageBytes;
    if (lane == 0) bulk_wait_group_read<1>();
    __syncwarp();
    const float *ws = s_ws + c * 32;
    const uint16_t *bs = s_bias + c * 32;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const float4 w0 = *reinterpret_cast<const float4 *>(ws + 8 * g);
      const float4 w1 = *reinterpret_cast<const float4 *>(ws + 8 * g + 4);
      float t[8];
      t[0] = dequant((int32_t)v[8 * g + 0], as, w0.x);
      t[1] = dequant((int32_t)v[8 * g + 1], as, w0.y);
      t[2] = dequant((int32_t)v[8 * g + 2], as, w0.z);
      t[3] = dequant((int32_t)v[8 * g + 3], as, w0.w);
      t[4] = dequant((int32_t)v[8 * g + 4], as, w1.x);
      t[5] = dequant((int32_t)v[8 * g + 5], as, w1.y);
      t[6] = dequant((int32_t)v[8 * g + 6], as, w1.z);
      t[7] = dequant((int32_t)v[8 * g + 7], as, w1.w);
      if (a.bias) {
        const uint4 b = *reinterpret_cast<const uint4 *>(bs + 8 * g);
        const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          t[2 * h] = __fadd_rn(t[2 * h], __uint_as_float(bw[h] << 16));
          t[2 * h + 1] = __fadd_rn(t[2 * h + 1], __uint_as_float(bw[h] & 0xFFFF0000u));
        }
      }
      if (a.act != W8A8_ACT_NONE) {
#pragma unroll
        for (int h = 0; h < 8; ++h) t[h] = apply_act(t[h], a.act);
      }
      *reinterpret_cast<uint4 *>(buf + swz64_offset(lane, g)) =
          make_uint4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]), pack_bf16x2(t[4], t[5]),
                     pack_bf16x2(t[6], t[7]));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(tmap_y, buf, n0, row_base + quarter * 32);
      bulk_commit_group();
    }
    ++stage_count;
  }
}

struct NoExtra {
  __device__ int operator()(int, int) const { return 0; }
};

}  // namespace w8a8
