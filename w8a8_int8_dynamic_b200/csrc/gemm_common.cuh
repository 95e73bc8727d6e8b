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
#include "quant_common.cuh"

namespace w8a8 {

constexpr int kBM = 128;                 // tile rows (MMA M)
constexpr int kBK = 128;                 // bytes of K per pipeline stage
constexpr int kTileBytes = 128 * kBK;    // one 128 x 128 int8 tile = 16 KB
constexpr int kThreads = 192;            // small-M kernel: 6 warps
constexpr int kDecodeNT = 16;            // activation rows per decode MMA (N)
// Large-M kernels: warp 1 MMA issuer, warps 2..9 epilogue, warp 0 idle, and
// the producer alone in an eleventh, one-thread warp (block kGemmThreads + 1).
// A warp may only read the TMEM lanes of its quarter (warp id mod 4), so the
// eight epilogue warps form two per lane quarter, each draining half of the
// tile's columns: two warps per SM sub-partition hide each other's latency.
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
// Register cap of the large-M GEMM kernels: 128 x 32 x 11 warps = 45,056 of an
// SM's 65,536 registers.  The 20,480 left hold four 4-warp quantisation
// blocks of 40 registers on paper; measured, a GEMM CTA starts early on SMs
// that hold three of them (most SMs, for 512 rows of 4096), not on those with
// four.
constexpr int kGemmRegs = 128;

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
  // 1-SM kernel: k-blocks of its first weight slab past the first stages that
  // a CTA asks L2 to fetch before waiting for the preceding kernel (0: none)
  int prefetch_kb;
  // pair kernel, whole tiles: tiles [0, full_tiles) run whole, each later one
  // as its two 128-column halves (a short last round spread over more pairs)
  int full_tiles;
  int row_major;  // tile order (tile_coords)
  int *status;
  // Next-layer quantisation fused with this layer (the kernels' ROWMAX
  // instances): the epilogue folds each row's largest bf16 output magnitude
  // into row_amax (atomicMax on the bf16 magnitude bits; zeroed by the
  // quantisation kernel ahead of this GEMM), and once a warp's output stores
  // for a tile are complete it adds the columns it stored to its 128-row
  // block's word in row_done ((done_tag << 32) | columns; a block is complete
  // at 4 N).  The kernel's own warps then form the codes q_next [M, N] and
  // scales a_scale_next [M] of each complete block (see codes_* below);
  // exit_word counts the CTAs out (the last one clears the block words for
  // the next call).
  uint32_t *row_amax;
  unsigned long long *row_done;
  unsigned long long done_tag;
  int8_t *q_next;
  float *a_scale_next;
  unsigned long long *exit_word;
};

// After a tile: the epilogue warp that drained rows [row0, row0 + 32) and
// `cols` of their columns (at least 1) publishes them to the codes kernel.
// Callers skip warps whose 128-row block lies wholly past M (no word exists
// for it); every warp of an existing block arrives, rows past M included, so
// that each block's count reaches 4 N.
// Each lane folds its row's maximum magnitude (bf16 magnitude bits) into
// row_amax; lane 0 waits
// until the warp's TMA stores of the tile have completed, orders them (async
// proxy) and the lanes' maxima before its arrival on the row block's word.
__device__ __forceinline__ void publish_rows(const GemmArgs &a, int lane, int row0,
                                             uint32_t max_bits, int cols) {
  const int row = row0 + lane;
  if (row < a.M) atomicMax(a.row_amax + row, max_bits);
  __threadfence();
  __syncwarp();
  if (lane == 0) {
    bulk_wait_group_all();
    fence_proxy_async_global();
    __threadfence();
    arrive_tagged32(a.row_done + (row0 >> 7), a.done_tag, (uint32_t)cols);
  }
  __syncwarp();
}

// The (row tile, column tile) of a linear tile index.  Plain instances walk
// the tiles column tile by column tile (row tile fastest: tiles running at
// the same time share a weight slab in L2, and each wave of tiles reads all
// of q again), or, with row_major, row tile by row tile (each wave reads all
// of the weights again).  ROWMAX instances walk them row tile by row tile,
// so that their row blocks complete one after another while the GEMM runs
// and the codes kernel beside it can follow.
template <bool ROWMAX>
__device__ __forceinline__ void tile_coords(const GemmArgs &a, int tile, int &mb, int &nb) {
  if (ROWMAX || a.row_major) {
    mb = tile / a.tiles_n;
    nb = tile - mb * a.tiles_n;
  } else {
    nb = tile / a.tiles_m;
    mb = tile - nb * a.tiles_m;
  }
}

// Epilogue warp ew (0..7): TMEM lane quarter and which half of the columns.
struct EpiWarp {
  int quarter, half;
  __device__ explicit EpiWarp(int warp) : quarter(warp & 3), half((warp - 2) >> 2) {}
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 r = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&r);
}

__device__ __forceinline__ float dequant(int32_t acc, float as, float ws) {
  return __fmul_rn(__fmul_rn(__int2float_rn(acc), as), ws);
}

// Stages the per-column scale and bias of COLS columns starting at global
// column n0 into the warp's own smem slice (all lanes then read them as
// broadcasts).  Columns past N read as zero.
template <int COLS>
__device__ __forceinline__ void stage_columns(const GemmArgs &a, int n0, int lane, float *s_ws,
                                              uint16_t *s_bias) {
#pragma unroll
  for (int j = lane * 4; j < COLS; j += 128) {
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n0 + j < a.N) v = __ldg(reinterpret_cast<const float4 *>(a.w_scale + n0 + j));
    *reinterpret_cast<float4 *>(s_ws + j) = v;
  }
  if (a.bias) {
#pragma unroll
    for (int j = lane * 8; j < COLS; j += 256) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n0 + j < a.N) v = __ldg(reinterpret_cast<const uint4 *>(a.bias + n0 + j));
      *reinterpret_cast<uint4 *>(s_bias + j) = v;
    }
  }
}

// The scale / bias / activation arithmetic of 8 consecutive columns of one
// row, in the defined order, packed to bf16 pairs.
__device__ __forceinline__ uint4 epilogue8(const GemmArgs &a, const uint32_t *v, float as,
                                           const float *ws, const uint16_t *bs) {
  const float4 w0 = *reinterpret_cast<const float4 *>(ws);
  const float4 w1 = *reinterpret_cast<const float4 *>(ws + 4);
  float t[8];
  t[0] = dequant((int32_t)v[0], as, w0.x);
  t[1] = dequant((int32_t)v[1], as, w0.y);
  t[2] = dequant((int32_t)v[2], as, w0.z);
  t[3] = dequant((int32_t)v[3], as, w0.w);
  t[4] = dequant((int32_t)v[4], as, w1.x);
  t[5] = dequant((int32_t)v[5], as, w1.y);
  t[6] = dequant((int32_t)v[6], as, w1.z);
  t[7] = dequant((int32_t)v[7], as, w1.w);
  if (a.bias) {
    const uint4 b = *reinterpret_cast<const uint4 *>(bs);
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      t[2 * h] = __fadd_rn(t[2 * h], __uint_as_float(bw[h] << 16));
      t[2 * h + 1] = __fadd_rn(t[2 * h + 1], __uint_as_float(bw[h] & 0xFFFF0000u));
    }
  }
  if (a.act != W8A8_ACT_NONE) {
#pragma unroll
    for (int h = 0; h < 4; ++h) apply_act_pair(t[2 * h], t[2 * h + 1], a.act);
  }
  return make_uint4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]), pack_bf16x2(t[4], t[5]),
                    pack_bf16x2(t[6], t[7]));
}

// Runs body(v, c) over the NCH 32-column chunks of a TMEM range, with the
// load of chunk c + 1 in flight while chunk c is processed.  `taddr` is the
// range's first column in this warp's lane quarter; `valid(c)` must be
// uniform across the warp and monotone (once false, false for later c).
template <int NCH, typename Valid, typename Body>
__device__ __forceinline__ void for_tmem_chunks(uint32_t taddr, Valid valid, Body body) {
  static_assert(NCH % 2 == 0, "chunks are processed in pairs");
  uint32_t v0[32], v1[32];
  if (!valid(0)) return;
  tmem_ld_32x32b_x32(taddr, v0);
#pragma unroll
  for (int c = 0; c < NCH; c += 2) {
    tmem_ld_wait_regs(v0);
    const bool more1 = valid(c + 1);
    if (more1) tmem_ld_32x32b_x32(taddr + (c + 1) * 32, v1);
    body(v0, c);
    __syncwarp();  // converged for the next .sync.aligned tcgen05 instruction
    if (!more1) return;
    tmem_ld_wait_regs(v1);
    const bool more2 = c + 2 < NCH && valid(c + 2);
    if (more2) tmem_ld_32x32b_x32(taddr + (c + 2) * 32, v0);
    body(v1, c + 1);
    __syncwarp();
    if (!more2) return;
  }
}

// As for_tmem_chunks, one chunk in flight at a time.
template <int NCH, typename Valid, typename Body>
__device__ __forceinline__ void for_tmem_chunks_single(uint32_t taddr, Valid valid, Body body) {
  uint32_t v[32];
#pragma unroll 1
  for (int c = 0; c < NCH; ++c) {
    if (!valid(c)) return;
    tmem_ld_32x32b_x32(taddr + c * 32, v);
    tmem_ld_wait_regs(v);
    body(v, c);
    __syncwarp();  // converged for the next .sync.aligned tcgen05 instruction
  }
}

// int32 accumulators straight to global memory (inspection export): COLS
// columns of this warp's 32 rows, starting at global column n0.
template <int COLS>
__device__ __forceinline__ void epilogue_i32(const GemmArgs &a, uint32_t taddr, int row, int n0) {
  const bool row_ok = row < a.M;
  for_tmem_chunks<COLS / 32>(
      taddr, [&](int c) { return n0 + c * 32 < a.N; },
      [&](const uint32_t(&v)[32], int c) {
        if (!row_ok) return;
        const int nc = n0 + c * 32;
        int32_t *dst = static_cast<int32_t *>(a.out) + (int64_t)row * a.N + nc;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (nc + 4 * g < a.N)
            *reinterpret_cast<uint4 *>(dst + 4 * g) =
                make_uint4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
      });
}

// Output staging for the TMA-store epilogue: each epilogue warp owns one
// 2 KB box, 32 rows x 32 bf16 columns in the 64-byte-swizzle layout of the
// output tensor map (16-byte chunk c of row r at chunk position
// c ^ ((r >> 1) & 3)), so the 32 lanes' 16-byte writes spread over all banks.
constexpr int kEpiStageBytes = 32 * 32 * 2;
constexpr int kEpiStagePerWarp = kEpiStageBytes;

// ---- the next layer's codes, formed by the fused GEMM's own warps ------------
// A unit is one row x kCodesSlice columns of the output, handled by one warp
// (each lane kCodesCPL 16-byte chunks, all loads in flight together), with
// the arithmetic of the quantisation kernel (quant_common.cuh) on the row's
// maximum from row_amax.  The units are dealt out in advance: of the W
// codes workers of the grid (warp 0 and the eight epilogue warps of every
// CTA), worker w takes units w, w + W, w + 2W, ... in that order, so that
// handing out work costs no atomics and each unit costs one round trip to
// learn that its row block is complete.  Warp 0, otherwise idle, waits for
// each block in turn; the epilogue warps take their next unit only if its
// block is already complete, in the gaps between their tiles, and after
// their last tile finish their share.  Rows are read through L2 only (.cg):
// other CTAs of the grid write them.
constexpr int kCodesCPL = 8;
constexpr int kCodesSlice = 32 * kCodesCPL * 8;  // 2048 columns
constexpr int kCodesWorkers = 1 + kEpiWarps;     // per CTA

__device__ __forceinline__ uint4 ld_cg_u4(const void *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ int codes_slices(const GemmArgs &a) {
  return (a.N + kCodesSlice - 1) / kCodesSlice;
}
__device__ __forceinline__ unsigned long long codes_want(const GemmArgs &a) {
  return (a.done_tag << 32) | (unsigned long long)(4 * a.N);
}

// A warp's share of the units: its next unit and the stride.
struct CodesCursor {
  uint32_t u, stride, units;
};
// worker: 0 for warp 0, 1 + e for epilogue warp e.
__device__ __forceinline__ CodesCursor codes_cursor(const GemmArgs &a, int worker) {
  CodesCursor c;
  c.stride = gridDim.x * (uint32_t)kCodesWorkers;
  c.u = blockIdx.x * (uint32_t)kCodesWorkers + (uint32_t)worker;
  c.units = (uint32_t)a.M * (uint32_t)codes_slices(a);
  return c;
}

// Waits until *word == want (acquire, every lane), the pause between reads
// doubling from 128 ns to 2 us: a row block completes every few
// microseconds, and many warps wait on the same word, whose L2 slice the
// GEMM's own traffic also uses.  The blocks are completed by CTAs of this
// grid, which is a single wave (at most one CTA or CTA pair per SM), so the
// wait ends unless something failed; it gives up like mbar_wait_bounded.
__device__ __forceinline__ bool wait_block(const unsigned long long *word, unsigned long long want,
                                           volatile int *abort_flag, int *status) {
  if (ld_acquire_gpu(word) == want) return true;
  const uint64_t t0 = global_timer_ns();
  unsigned pause = 128;
  while (true) {
    __nanosleep(pause);
    if (pause < 2048) pause *= 2;
    if (ld_acquire_gpu(word) == want) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      atomicExch(status, (int)W8A8_ERR_TIMEOUT);
      return false;
    }
  }
}

// Unit u, whose row block every lane has acquired complete, by the warp.
__device__ __forceinline__ void codes_unit(const GemmArgs &a, uint32_t u, int lane) {
  const int slices = codes_slices(a);
  const int row = (int)(u / (uint32_t)slices);
  const int slice = (int)(u - (uint32_t)row * (uint32_t)slices);
  const uint16_t *yr = static_cast<const uint16_t *>(a.out) + (int64_t)row * a.N;
  int8_t *qr = a.q_next + (int64_t)row * a.N;
  const int nchunks = a.N >> 3;
  const int c0 = slice * (kCodesSlice / 8) + lane;
  uint4 v[kCodesCPL];
#pragma unroll
  for (int j = 0; j < kCodesCPL; ++j) {
    const int c = c0 + 32 * j;
    v[j] = make_uint4(0, 0, 0, 0);
    if (c < nchunks) v[j] = ld_cg_u4(yr + (int64_t)c * 8);
  }
  const float amax = __uint_as_float(__ldcg(a.row_amax + row) << 16);
  const float s = amax == 0.0f ? 0.0f : __fdiv_rn(amax, 127.0f);
  if (slice == 0 && lane == 0) a.a_scale_next[row] = s;
  if (amax == 0.0f) {
#pragma unroll
    for (int j = 0; j < kCodesCPL; ++j) {
      const int c = c0 + 32 * j;
      if (c < nchunks) *reinterpret_cast<uint2 *>(qr + (int64_t)c * 8) = make_uint2(0, 0);
    }
  } else if (s >= 1e-30f) {
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int j = 0; j < kCodesCPL; ++j) {
      const int c = c0 + 32 * j;
      if (c < nchunks) *reinterpret_cast<uint2 *>(qr + (int64_t)c * 8) = codes8(v[j], s, inv);
    }
  } else {
    // (unrolled: a runtime index into v would move it to local memory)
#pragma unroll
    for (int j = 0; j < kCodesCPL; ++j) {
      const int c = c0 + 32 * j;
      if (c < nchunks) *reinterpret_cast<uint2 *>(qr + (int64_t)c * 8) = codes8_ieee(v[j], s);
    }
  }
}

// The warp's next unit, if any.  blocking: wait (bounded) for its row block;
// otherwise only if the block is already complete.  False: none processed
// (blocking: the share is done, or abort).
__device__ __forceinline__ bool codes_next(const GemmArgs &a, int lane, CodesCursor &c,
                                           bool blocking, volatile int *abort_flag) {
  if (c.u >= c.units) return false;
  const int slices = codes_slices(a);
  const unsigned long long *word = a.row_done + ((c.u / (uint32_t)slices) >> 7);
  if (blocking) {
    if (!wait_block(word, codes_want(a), abort_flag, a.status)) {
      c.u = c.units;  // abort: stop
      return false;
    }
  } else if (ld_acquire_gpu(word) != codes_want(a)) {
    return false;
  }
  (void)lane;
  codes_unit(a, c.u, lane);
  c.u += c.stride;
  return true;
}

// An epilogue warp about to wait for its next tile's accumulators forms codes
// of complete row blocks while they are not ready yet.
__device__ __forceinline__ void codes_while_waiting(const GemmArgs &a, int lane, CodesCursor &c,
                                                    uint64_t *tfull, uint32_t parity) {
  while (true) {
    int ready = 0;
    if (lane == 0) ready = mbar_try_wait(smem_addr(tfull), parity) ? 1 : 0;
    ready = __shfl_sync(0xFFFFFFFFu, ready, 0);
    if (ready || !codes_next(a, lane, c, false, nullptr)) return;
  }
}

// After the CTA's last barrier: thread 0 counts the CTA out; the last CTA of
// the grid clears the block words (every CTA is past its waits), so that a
// replayed CUDA graph, which keeps the tag, starts from zero.
__device__ __forceinline__ void codes_exit(const GemmArgs &a) {
  __shared__ int last_cta;
  if (threadIdx.x == 0) {
    __threadfence();
    last_cta = arrive_tagged32(a.exit_word, a.done_tag, 1u) == gridDim.x ? 1 : 0;
  }
  __syncthreads();
  if (last_cta) {
    const int nblk = (a.M + 127) >> 7;
    for (int b = threadIdx.x; b < nblk; b += blockDim.x) a.row_done[b] = 0ull;
    if (threadIdx.x == 0) *a.exit_word = 0ull;
  }
}

// The two packed 16-bit magnitudes of epilogue_tma's rmax -> one bf16
// magnitude bit pattern (finite bf16 order by magnitude = order of these bits).
__device__ __forceinline__ uint32_t row_max_bits(uint32_t rmax) {
  return max(rmax & 0xFFFFu, rmax >> 16);
}

__device__ __forceinline__ uint32_t swz64_offset(int r, int c16) {
  return (uint32_t)(r * 64 + ((c16 ^ ((r >> 1) & 3)) << 4));
}

// Drains COLS accumulator columns of this warp's 32 rows from TMEM and
// writes them as bf16 through shared memory, one TMA store per 32 x 32 box
// (rows and columns outside the output are clipped by the tensor map).
//   taddr   TMEM address of the first column, this warp's lane quarter
//   row0    output row of lane 0;  n0: output column of the first column
//   s_ws / s_bias: the COLS columns' scales and bias, staged in smem
//   rmax    (ROWMAX) the running maximum of this lane's row's bf16 output
//           magnitudes, as two packed 16-bit lanes (see row_max_bits)
//   ncols   columns actually drained (a multiple of 32, at most COLS)
template <int COLS, bool ROWMAX>
__device__ __forceinline__ void epilogue_tma(const GemmArgs &a, const CUtensorMap *tmap_y,
                                             uint32_t taddr, int lane, int row0, int n0, float as,
                                             const float *s_ws, const uint16_t *s_bias,
                                             uint8_t *stage, uint32_t &rmax, int ncols = COLS) {
  // ROWMAX instances load one chunk at a time: their tiles are long (large
  // M, N and K), so the epilogue is far off the critical path, and the
  // registers of the second chunk buffer leave room beside the GEMM for the
  // codes kernel's warps.
  auto run = [&](auto valid, auto body) {
    if (ROWMAX)
      for_tmem_chunks_single<COLS / 32>(taddr, valid, body);
    else
      for_tmem_chunks<COLS / 32>(taddr, valid, body);
  };
  run([&](int c) { return c * 32 < ncols && n0 + c * 32 < a.N; },
      [&](const uint32_t(&v)[32], int c) {
        uint4 out[4];
#pragma unroll
        for (int g = 0; g < 4; ++g)
          out[g] = epilogue8(a, v + 8 * g, as, s_ws + c * 32 + 8 * g, s_bias + c * 32 + 8 * g);
        if (ROWMAX) {
          // Columns past N hold exact zeros (zero weights, scale and bias).
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            rmax = __vmaxu2(rmax, out[g].x & 0x7FFF7FFFu);
            rmax = __vmaxu2(rmax, out[g].y & 0x7FFF7FFFu);
            rmax = __vmaxu2(rmax, out[g].z & 0x7FFF7FFFu);
            rmax = __vmaxu2(rmax, out[g].w & 0x7FFF7FFFu);
          }
        }
        // the box was last read by this warp's previous store
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
#pragma unroll
        for (int g = 0; g < 4; ++g) *reinterpret_cast<uint4 *>(stage + swz64_offset(lane, g)) = out[g];
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(tmap_y, stage, n0 + c * 32, row0);
          bulk_commit_group();
        }
      });
}

}  // namespace w8a8
