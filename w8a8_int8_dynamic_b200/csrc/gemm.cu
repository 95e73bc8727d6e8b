// gemm.cu -- int8 x int8 -> int32 GEMM on the sm_100a tensor cores with the
// dequantising epilogue; the kernel choice for large M; and the C entry points
// of the GEMM and of the whole layer (quantisation kernel, then the GEMM as a
// programmatic dependent launch).
//
// Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
// Round two: the cutlass_scaled_mm op (int8 activations x int8 weights,
// per-token and per-output-channel fp32 scales, bf16 out), fused Q/K/V and
// row-parallel layer shapes.  "INT8 Quant for Dual-Max Recipe": W8A8 runs
// int8 x int8 natively on the integer tensor cores, weights never
// dequantised; prefill is compute-bound, decode is weight-bandwidth-bound.
//
//   acc[m,n] = sum_k q[m,k] w[n,k]                     (exact int32, TMEM)
//   y[m,n]   = bf16_rne(((float)acc * a_scale[m]) * w_scale[n] + bias[n])
//
// 1. gemm_kernel (large M): persistent, one CTA per SM, 321 threads of at
//    most 128 registers (room for quantisation CTAs beside it).
//    thread 320, alone in the last warp: producer -- per stage of KPS
//            k-blocks, TMA 2-D loads of the q tiles (128 rows x 128 bytes,
//            128-byte swizzle) and one bulk copy
//            of the KPS contiguous weight tiles of each 128-row slab from the
//            packed image, onto a STAGES-deep mbarrier ring; a cursor keeps
//            the address arithmetic out of the slot turnaround.  Behind the
//            quantisation kernel it first issues the weight copies of the
//            first stages, waits for the codes, then asks L2 to prefetch
//            more of its slab;
//    warp 1: MMA issuer -- 4 x tcgen05.mma.kind::i8 (M=128, N=BN, K=32) per
//            k-block, int32 accumulators in TMEM, double-buffered so the
//            epilogue of tile i overlaps the main loop of tile i+1;
//    warps 2-9: epilogue -- two warps per TMEM lane quarter, half the columns
//            each; tcgen05.ld of 32 columns at a time with the next load in
//            flight, the scale / bias (/ GELU) arithmetic in fp32 (each step
//            rounded separately, so the result is bit-identical to the
//            definition), bf16 through swizzled shared-memory boxes and TMA
//            stores.
// 2. The 2-SM pair kernel (gemm2sm.cu) and the small-M weight-streaming
//    kernel (decode.cu) share the tile image and epilogue arithmetic.
//
// Every mbarrier wait is time-bounded (ptx.cuh); a wait that gives up sets
// the device status word to W8A8_ERR_TIMEOUT and the block drains and exits.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "gemm_common.cuh"

namespace w8a8 {
namespace {

// ============================================================================
// Large-M persistent GEMM
// ============================================================================
// KPS = k-blocks per pipeline stage.  With 128-wide tiles the KPS weight
// tiles of a stage are contiguous in the packed image (one bulk copy); fewer,
// larger stages halve the per-stage barrier round trips that bound the feed.
template <int BN, int STAGES, int KPS>
struct LargeSmem {
  static constexpr int kAStage = KPS * kTileBytes;
  static constexpr int kBStage = KPS * BN * kBK;
  static constexpr int kA = 0;
  static constexpr int kB = STAGES * kAStage;
  // per epilogue warp: its BN/2 columns' w_scale (fp32) and bias (bf16) values
  static constexpr int kEpiPerWarp = (BN / 2) * 6;
  static constexpr int kEpi = kB + STAGES * kBStage;
  static constexpr int kEpiEnd = kEpi + kEpiWarps * kEpiPerWarp;
  static constexpr int kOut = kEpiEnd + 1024 - kEpiEnd % 1024;
  static constexpr int kBars = kOut + kEpiWarps * kEpiStagePerWarp;  // full[S], empty[S], tfull[2], tempty[2], done
  static constexpr int kMisc = kBars + (2 * STAGES + 5) * 8;
  static constexpr int kUsed = kMisc + 16;
  static constexpr int kAlloc = kUsed + 1024;  // slack for 1024-byte alignment
  static_assert(KPS == 1 || BN == 128, "multi-k-block stages need contiguous weight tiles");
};

// At most kGemmRegs registers a thread, so that a CTA (11 warps) fits on an
// SM beside the blocks of the quantisation kernel it is launched behind and
// starts its prologue and first weight copies while they run.
// ROWMAX: the next layer's quantisation is fused in (GemmArgs::row_amax).
template <int BN, int STAGES, int KPS, bool OUT_I32, bool ROWMAX>
__global__ void __maxnreg__(kGemmRegs)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_q,
                const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
  using L = LargeSmem<BN, STAGES, KPS>;
  constexpr uint32_t kTmemCols = 2 * BN;  // two accumulator buffers
  constexpr uint32_t kIdesc = idesc_i8(kBM, BN);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem + L::kA;
  uint8_t *sB = smem + L::kB;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBars);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *mma_done = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

  // With the next layer's quantisation fused in, the next layer's GEMM (a
  // programmatic dependent) takes each SM as this kernel leaves it.
  if (ROWMAX) griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmap_q);
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = args.tiles_m * args.tiles_n;
  const int num_kb = args.num_kb;
  const int nsk = (num_kb + KPS - 1) / KPS;  // stages per tile
  const int my_tiles = blockIdx.x < num_tiles ? (num_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  const uint32_t my_iters = (uint32_t)my_tiles * nsk;

  // Roles: the producer is the lone thread of a last, one-thread warp (block
  // = kGemmThreads + 1).  With no other lane of its warp parked at a
  // barrier, its wait-then-copy loop turns a stage around sooner: a scratch
  // microbenchmark streams 32 KB bulk copies at 141 GB/s per SM from such a
  // thread against 126 GB/s from lane 0 of a warp whose other lanes wait at
  // __syncwarp, and the square GEMM runs 4 % faster.  Lane 0 of warp 1 runs
  // the MMA loop alone (the rest of warp 1 waits at __syncwarp so the warp
  // reaches the block barrier below converged; the warp also owns the TMEM
  // allocation); warp 0 is idle.
  if (threadIdx.x == kGemmThreads) {
    // ---------------- producer ----------------
    // A cursor walks this CTA's stages in order; the divisions by runtime
    // tile counts and the 64-bit slab offsets are taken once per tile, after
    // a stage's copies are issued.  Between a slot's release and its refill
    // only the copies themselves remain: the issuing thread is on the ring's
    // critical path (a scratch microbenchmark of 64 KB stages moves 118 GB/s
    // per SM with a 64-bit modulo per stage in that thread, 170 GB/s without).
    const size_t slab_bytes = (size_t)num_kb * kTileBytes;  // one 128-row weight slab
    struct Cursor {
      int tile, j, q_row;       // tile index, stage within the tile, first q row
      const uint8_t *w;         // the tile's first weight slab
    };
    auto at_tile = [&](int tile) {
      Cursor c;
      c.tile = tile;
      c.j = 0;
      int mb, nb;
      tile_coords<ROWMAX>(args, tile, mb, nb);
      c.q_row = mb * kBM;
      c.w = args.packed_w + (size_t)nb * (BN / 128) * slab_bytes;
      return c;
    };
    auto advance = [&](Cursor &c) {
      if (++c.j == nsk) c = at_tile(c.tile + (int)gridDim.x);
    };
    auto stage_nk = [&](const Cursor &c) { return min(KPS, num_kb - c.j * KPS); };
    auto weights = [&](const Cursor &c, uint32_t s, int nk) {
      const uint8_t *src = c.w + (size_t)(c.j * KPS) * kTileBytes;
#pragma unroll
      for (int h = 0; h < BN / 128; ++h)
        bulk_load(sB + s * L::kBStage + h * kTileBytes, src + h * slab_bytes,
                  (uint32_t)(nk * kTileBytes), &full[s]);
    };
    auto acts = [&](const Cursor &c, uint32_t s, int nk) {
      for (int i = 0; i < nk; ++i)
        tma_load_2d(sA + s * L::kAStage + i * kTileBytes, &tmap_q, (c.j * KPS + i) * kBK, c.q_row,
                    &full[s]);
    };
    constexpr uint32_t kBytesPerKb = kTileBytes + BN * kBK;
    const uint32_t pre = my_iters < (uint32_t)STAGES ? my_iters : (uint32_t)STAGES;
    if (my_tiles > 0) {
      Cursor cur = at_tile(blockIdx.x);
      // The weight tiles of the first stages do not depend on the preceding
      // kernel of the stream: issue them before waiting for it.
      const Cursor first = cur;
      for (uint32_t it = 0; it < pre; ++it) {
        const int nk = stage_nk(cur);
        mbar_arrive_expect_tx(&full[it], (uint32_t)nk * kBytesPerKb);
        weights(cur, it, nk);
        advance(cur);
      }
      griddep_wait();
      if (args.prefetch_kb > 0) {
        // CTAs blockIdx.x / tiles_m read the same slab: each warms its share.
        // Issued after the wait: with the CTA resident beside the
        // quantisation blocks, prefetches in flight when they finish delay
        // the release of the wait (square layer 15.9 -> 15.6 us).
        const int mb = blockIdx.x % args.tiles_m;
        const int kb_lo = STAGES * KPS, kb_hi = min(num_kb, kb_lo + args.prefetch_kb);
        if (kb_hi > kb_lo) {
          const int per = (kb_hi - kb_lo + args.tiles_m - 1) / args.tiles_m;
          const int k0 = kb_lo + mb * per, k1 = min(kb_hi, k0 + per);
          if (k1 > k0)
#pragma unroll
            for (int h = 0; h < BN / 128; ++h)
              bulk_prefetch_l2(first.w + h * slab_bytes + (size_t)k0 * kTileBytes,
                               (uint32_t)((k1 - k0) * kTileBytes));
        }
      }
      {
        Cursor c = first;
        for (uint32_t it = 0; it < pre; ++it) {
          acts(c, it, stage_nk(c));
          advance(c);
        }
      }
      uint32_t issued = pre, s = 0, ph = 1;  // stage `pre` (if any) reuses slot 0, second round
      bool ok = true;
      for (; issued < my_iters; ++issued) {
        const int nk = stage_nk(cur);
        const uint32_t bytes = (uint32_t)nk * kBytesPerKb;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], bytes);
        acts(cur, s, nk);
        weights(cur, s, nk);
        advance(cur);
        if (++s == (uint32_t)STAGES) {
          s = 0;
          ph ^= 1;
        }
      }
      if (!ok) {
        // Drain: wait (bounded) for the copies still in flight into our smem:
        // the last stage issued into each slot.
        for (uint32_t sl = 0; sl < (uint32_t)STAGES && sl < issued; ++sl) {
          const uint32_t last = sl + ((issued - 1 - sl) / STAGES) * STAGES;
          volatile int no_abort = 0;
          (void)mbar_wait_bounded(&full[sl], (last / STAGES) & 1, &no_abort, args.status);
        }
      }
    }
  } else if (warp == 0) {
    // idle, or (next-layer quantisation fused in) forming codes of the
    // output's row blocks as they complete
    if (ROWMAX) {
      CodesCursor cursor = codes_cursor(args, 0);
      while (codes_next(args, lane, cursor, true, abort_flag)) {
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      // Slot, phase and operand descriptors advance by counters, so a full
      // stage is answered by its MMAs at once.  A descriptor's address field
      // is the shared-memory address / 16, linear below 256 KB.
      const uint64_t a_desc0 = sw128_kmajor_desc(sA), b_desc0 = sw128_kmajor_desc(sB);
      uint32_t s = 0, ph = 0;
      bool ok = true;
      for (int t = 0; ok && t < my_tiles; ++t) {
        const uint32_t b = t & 1, bph = (t >> 1) & 1;
        if (!mbar_wait(&tempty[b], bph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int j = 0; j < nsk; ++j) {
          const int nk = min(KPS, num_kb - j * KPS);
          const uint64_t a_desc = a_desc0 + ((s * L::kAStage) >> 4);
          const uint64_t b_desc = b_desc0 + ((s * L::kBStage) >> 4);
          if (!mbar_wait(&full[s], ph, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int i = 0; i < nk; ++i) {
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_i8(d_tmem, a_desc + ((i * kTileBytes) >> 4) + 2 * k,
                     b_desc + ((i * BN * kBK) >> 4) + 2 * k, kIdesc, (j | i | k) != 0);
          }
          mma_commit(&empty[s]);  // frees the stage when these MMAs finish
          if (++s == (uint32_t)STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) mma_commit(&tfull[b]);
      }
      if (!ok) {
        // Wait (bounded) for MMAs still in flight before TMEM is released.
        mma_commit(mma_done);
        volatile int no_abort = 0;
        (void)mbar_wait_bounded(mma_done, 0, &no_abort, args.status);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    griddep_wait();  // a_scale comes from the preceding kernel
    constexpr int kCols = BN / 2;  // columns of the tile this warp drains
    const EpiWarp ew(warp);
    float *s_ws = reinterpret_cast<float *>(smem + L::kEpi + (warp - 2) * L::kEpiPerWarp);
    uint16_t *s_bias = reinterpret_cast<uint16_t *>(s_ws + kCols);
    uint8_t *s_out = smem + L::kOut + (warp - 2) * kEpiStagePerWarp;
    CodesCursor cursor = codes_cursor(args, warp - 1);  // (ROWMAX) this warp's codes units
    for (int t = 0; t < my_tiles; ++t) {
      const int tile = blockIdx.x + t * gridDim.x;
      int mb, nb;
      tile_coords<ROWMAX>(args, tile, mb, nb);
      const uint32_t b = t & 1, bph = (t >> 1) & 1;
      const int n0 = nb * BN + ew.half * kCols;
      const int row0 = mb * kBM + ew.quarter * 32;
      // operands of the epilogue, fetched while the main loop runs
      float as = 0.0f;
      if (!OUT_I32) {
        stage_columns<kCols>(args, n0, lane, s_ws, s_bias);
        if (row0 + lane < args.M) as = __ldg(args.a_scale + row0 + lane);
      }
      __syncwarp();
      if (ROWMAX) codes_while_waiting(args, lane, cursor, &tfull[b], bph);
      int ok = 0;
      if (lane == 0) ok = mbar_wait(&tfull[b], bph, abort_flag, args.status);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + b * BN + ew.half * kCols + ((uint32_t)(ew.quarter * 32) << 16);
      uint32_t rmax = 0;
      if (OUT_I32)
        epilogue_i32<kCols>(args, taddr, row0 + lane, n0);
      else
        epilogue_tma<kCols, ROWMAX>(args, &tmap_y, taddr, lane, row0, n0, as, s_ws, s_bias, s_out,
                                    rmax);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);
      if (ROWMAX && n0 < args.N && (row0 >> 7) * 128 < args.M)
        publish_rows(args, lane, row0, row_max_bits(rmax), min(kCols, args.N - n0));
    }
    if (lane == 0) bulk_wait_group_all();  // output stores complete before exit
    __syncwarp();
    if (ROWMAX)  // help with the codes still to form
      while (codes_next(args, lane, cursor, true, abort_flag)) {
      }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
  if (ROWMAX) codes_exit(args);
}

// ============================================================================
// host side
// ============================================================================
constexpr int kLargeStages128 = 3;  // 3 x (2 k-blocks): 64 KB stages
constexpr int kKps128 = 2;
// When the GEMM follows the activation quantisation in the same stream, that
// kernel leaves DRAM mostly idle: the GEMM's CTAs, resident beside it, ask L2
// for the next 32 k-blocks of their weight slab (512 KB per 128-row slab,
// shared out among the CTAs that read the slab) before they wait for the
// codes.  Measured on 512 x 4096 x K: the layer step 18.0 -> 17.25 us at
// K = 4096, 29.7 -> 29.2 us at K = 8192.  Prefetching the whole slab was
// slower at K = 8192 (30.6 us), and a standalone GEMM (nothing to overlap
// with) runs slower with any prefetch, so it takes none.
constexpr int kPrefetchKb = 32;
constexpr int kLargeStages256 = 4;  // 4 x (1 k-block): 48 KB stages

FuncAttrOnce g_smem_attr[8];  // one per kernel instance (`slot`)

template <typename Kernel>
cudaError_t set_smem_attr(Kernel k, int bytes, int slot) {
  return g_smem_attr[slot].ensure(
      [&] { return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes); });
}

template <typename Kernel, typename... Args>
cudaError_t launch_ex(Kernel k, int grid, int smem, cudaStream_t stream, bool pdl,
                      const Args &...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kGemmThreads + 1);  // + the producer's one-thread warp
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

template <int BN, int STAGES, bool OUT_I32, bool ROWMAX = false>
w8a8_status run_large(const CUtensorMap &tmap, const CUtensorMap &tmap_y, GemmArgs args,
                      cudaStream_t stream, bool pdl, int slot) {
  constexpr int KPS = BN == 128 ? kKps128 : 1;
  using L = LargeSmem<BN, STAGES, KPS>;
  auto k = gemm_kernel<BN, STAGES, KPS, OUT_I32, ROWMAX>;
  cudaError_t e = set_smem_attr(k, L::kAlloc, slot);
  if (e != cudaSuccess) return W8A8_ERR_CUDA;
  args.tiles_n = (int)((args.N + BN - 1) / BN);
  const int tiles = args.tiles_m * args.tiles_n;
  const int grid = std::min(tiles, sm_count());
  e = launch_ex(k, grid, L::kAlloc, stream, pdl, tmap, tmap_y, args);
  count_launch();
  return from_cuda(e);
}

// Kernel choice for large M.  Per-SM feed from L2 limits how much of the
// int8 rate each tile shape reaches (measured: the 128 x 128 1-SM tile needs
// ~128 B/clk per SM, the 128 x 256 tile ~94, the 2-SM 256 x 256 tile ~64),
// so the cost of a shape is its wave count times its per-SM tile work divided
// by the fraction of the rate it sustains.
enum class LargeKind { k128, k256, kPair, kPair128 };

// Kernel choice for large M: (waves of tiles) x (per-SM time of one tile).
// The per-SM time of a stage of two k-blocks is set by what has to reach the
// SM (about 100-115 GB/s per SM in these kernels: stage slots of ~190 KB
// cycle through the loaded-L2 latency and the MMAs), by a whole-chip delivery
// term, or by the MMAs, whichever is slowest: 1-SM 128x128: 64 KB / 512
// cycles; 1-SM 128x256: 96 KB / 1024; pair 256x256: 64 KB / 1024; pair
// 256x128: 48 KB / 512 per SM.  The constants are calibrated against timings
// on this B200, not derived.
LargeKind choose_large(int64_t M, int64_t N) {
  const int path = forced_path();
  if (path == 3) return LargeKind::k128;
  if (path == 4) return LargeKind::k256;
  if (path == 5) return LargeKind::kPair;
  if (path == 7) return LargeKind::kPair128;
  const int64_t sms = sm_count(), pairs = sms / 2;
  const double feed_us_per_kb = 1.0 / 114e3;  // us per byte per SM
  const double l2_us_per_byte = 1.0 / 10.5e6;  // us per byte, whole chip
  const double mma_us_per_cycle = 1.0 / 1900.0;
  // one stage of every busy SM: per-SM feed, aggregate L2 and MMA bounds
  auto stage_us_on = [&](double bytes, double cycles, int64_t busy_sms) {
    return std::max({bytes * feed_us_per_kb, bytes * (double)busy_sms * l2_us_per_byte,
                     cycles * mma_us_per_cycle});
  };
  const int64_t tm = (M + kBM - 1) / kBM;
  const int64_t t128 = tm * ((N + 127) / 128), t256 = tm * ((N + 255) / 256);
  const int64_t tp256 = pair_tiles(M, N, 256), tp128 = pair_tiles(M, N, 128);
  auto cost = [&](int64_t tiles, int64_t slots, int ctas_per_tile, double bytes, double cycles) {
    const int64_t waves = (tiles + slots - 1) / slots;
    const int64_t busy = std::min(tiles, slots) * ctas_per_tile;
    return (double)waves * stage_us_on(bytes, cycles, busy);
  };
  const double c128 = cost(t128, sms, 1, 65536, 512);
  const double c256 = cost(t256, sms, 1, 98304, 1024);
  double cp256 = cost(tp256, pairs, 2, 65536, 1024);
  if (pair_full_tiles(tp256, pairs) < tp256)  // a short last round runs as half tiles
    cp256 -= 0.25 * cost(pairs, pairs, 2, 65536, 1024);
  const double cp128 = cost(tp128, pairs, 2, 49152, 512);
  // Few 256-wide pair tiles (half the GPU or less) but 128x128 tiles that fit
  // one wave: with cold operands, twice as many SMs pulling from DRAM wins
  // (measured on 512 x 4096 x 4096: 16.6 us vs 19.1 us for 256x256 pairs).
  if (tp256 * 2 <= pairs && t128 <= sms) return LargeKind::k128;
  double best = c128;
  LargeKind kind = LargeKind::k128;
  if (c256 < best) best = c256, kind = LargeKind::k256;
  if (cp256 <= best) best = cp256, kind = LargeKind::kPair;
  if (cp128 < best * 0.97) best = cp128, kind = LargeKind::kPair128;
  return kind;
}

}  // namespace

w8a8_status launch_scaled_mm(const int8_t *q, const float *a_scale, const void *packed_w,
                             const float *w_scale, const void *bias, void *out, bool out_i32,
                             int64_t M, int64_t N, int64_t K, cudaStream_t stream, bool pdl,
                             int act, bool prefetch, const RowSignal *sig) {
  CUtensorMap tmap;
  if (!make_tmap_u8_2d(&tmap, q, (uint64_t)M, (uint64_t)K, (uint64_t)K, kBM, kBK))
    return W8A8_ERR_CUDA;
  GemmArgs a{};
  a.packed_w = static_cast<const uint8_t *>(packed_w);
  a.a_scale = a_scale;
  a.w_scale = w_scale;
  a.bias = static_cast<const uint16_t *>(bias);
  a.out = out;
  a.M = (int)M;
  a.N = (int)N;
  a.num_kb = (int)(packed_cols(K) / 128);
  a.tiles_m = (int)((M + kBM - 1) / kBM);
  a.tiles_n = 0;
  a.act = out_i32 ? W8A8_ACT_NONE : act;
  // (the prefetch shares slabs out by the plain tile order)
  a.prefetch_kb = (pdl && prefetch && !sig) ? kPrefetchKb : 0;
  a.status = status_word();
  if (!a.status) return W8A8_ERR_CUDA;
  if (sig && !out_i32) {
    a.row_amax = sig->row_amax;
    a.row_done = sig->row_done;
    a.done_tag = sig->tag;
    a.q_next = sig->q_next;
    a.a_scale_next = sig->a_scale_next;
    a.exit_word = sig->exit_word;
  }
  CUtensorMap tmap_y;
  if (out_i32) {
    // the int32 export always uses the 1-SM kernel (tests and inspection); it
    // stores from registers and takes no output tensor map
    memset(&tmap_y, 0, sizeof(tmap_y));
    const LargeKind kind = choose_large(M, N);
    return kind == LargeKind::k128
               ? run_large<128, kLargeStages128, true>(tmap, tmap_y, a, stream, pdl, 1)
               : run_large<256, kLargeStages256, true>(tmap, tmap_y, a, stream, pdl, 0);
  }
  if (!make_tmap_out_bf16(&tmap_y, out, (uint64_t)M, (uint64_t)N)) return W8A8_ERR_CUDA;
  switch (choose_large(M, N)) {
    case LargeKind::kPair:
      return launch_gemm2sm(q, a_scale, packed_w, w_scale, bias, out, M, N, K, stream, pdl, 256,
                            act, sig);
    case LargeKind::kPair128:
      return launch_gemm2sm(q, a_scale, packed_w, w_scale, bias, out, M, N, K, stream, pdl, 128,
                            act, sig);
    case LargeKind::k256:
      return sig ? run_large<256, kLargeStages256, false, true>(tmap, tmap_y, a, stream, pdl, 4)
                 : run_large<256, kLargeStages256, false>(tmap, tmap_y, a, stream, pdl, 2);
    default:
      return sig ? run_large<128, kLargeStages128, false, true>(tmap, tmap_y, a, stream, pdl, 5)
                 : run_large<128, kLargeStages128, false>(tmap, tmap_y, a, stream, pdl, 3);
  }
}

// Largest N of the fused next-layer quantisation (a row block's completion
// count, 4 N, stays in 32 bits).
constexpr int64_t kMaxFusedN = (int64_t)1 << 28;

// Workspace of w8a8_linear_act_quant: as w8a8_linear's, then the row maxima,
// one completion word per 128-row block, and an exit word.
int64_t act_quant_workspace_bytes(int64_t M, int64_t N, int64_t K);

// Workspace of w8a8_linear: the codes, the scales and (small M) the split-K
// partials of the weight-streaming kernel.
int64_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  int64_t b = round_up(M * K, 256) + round_up(M * 4, 256);
  if (M <= kDecodeNT) b += decode_workspace_bytes(N, K);
  return b;
}

int64_t act_quant_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  return linear_workspace_bytes(M, N, K) + round_up(M * 4, 256) +
         round_up(((M + 127) / 128) * 8, 256) + 256;
}

static w8a8_status check_gemm_args(const void *q, const void *packed_w, const void *out,
                                   int64_t M, int64_t N, int64_t K) {
  if (!q || !packed_w || !out) return W8A8_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7FFFFFFF || N < 1 || K < 1) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0 || N > ((int64_t)1 << 30))
    return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q) || !aligned16(packed_w) || !aligned16(out)) return W8A8_ERR_ALIGNMENT;
  return W8A8_OK;
}

}  // namespace w8a8

using namespace w8a8;

extern "C" {

w8a8_status w8a8_scaled_mm_workspace_bytes(int64_t M, int64_t N, int64_t K, size_t *bytes) {
  if (!bytes || M < 1 || N < 1 || K < 1) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0) return W8A8_ERR_UNSUPPORTED_SHAPE;
  *bytes = (size_t)(M <= kDecodeNT ? decode_workspace_bytes(N, K) : 0);
  return W8A8_OK;
}

w8a8_status w8a8_scaled_mm_act(const int8_t *q, const float *a_scale, const void *packed_w,
                               const float *w_scale, const void *bias, void *y, int64_t M,
                               int64_t N, int64_t K, int act, void *workspace, size_t ws_bytes,
                               w8a8_stream_t stream) {
  w8a8_status st = check_gemm_args(q, packed_w, y, M, N, K);
  if (st != W8A8_OK) return st;
  if (!a_scale || !w_scale) return W8A8_ERR_INVALID_ARG;
  if (act != W8A8_ACT_NONE && act != W8A8_ACT_GELU_TANH) return W8A8_ERR_INVALID_ARG;
  if (!aligned16(a_scale) || !aligned16(w_scale) || (bias && !aligned16(bias)))
    return W8A8_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (use_decode_path(M) && workspace) {
    if (!aligned16(workspace)) return W8A8_ERR_ALIGNMENT;
    if ((int64_t)ws_bytes < decode_workspace_bytes(N, K)) return W8A8_ERR_BUFFER_TOO_SMALL;
    // A programmatic dependent, like the large-M path: back to back, each
    // launch streams its first weights while the previous one sums its last
    // slabs (M = 1..16 x 27648 x 5120: 30.1-30.9 -> 27.0-27.4 us a launch).
    return launch_decode(q, a_scale, packed_w, w_scale, bias, y, M, N, K, workspace, s, true,
                         act);
  }
  if (forced_path() == 2) return W8A8_ERR_INVALID_ARG;  // small path needs M <= 16 and a workspace
  if (workspace && !aligned16(workspace)) return W8A8_ERR_ALIGNMENT;
  // A programmatic dependent of the preceding kernel: behind the codes kernel
  // of a fused next-layer quantisation its CTAs take SMs as the previous
  // GEMM leaves them and issue their first weight copies while it finishes.
  return launch_scaled_mm(q, a_scale, packed_w, w_scale, bias, y, false, M, N, K, s, true, act);
}

w8a8_status w8a8_scaled_mm(const int8_t *q, const float *a_scale, const void *packed_w,
                           const float *w_scale, const void *bias, void *y, int64_t M, int64_t N,
                           int64_t K, void *workspace, size_t ws_bytes, w8a8_stream_t stream) {
  return w8a8_scaled_mm_act(q, a_scale, packed_w, w_scale, bias, y, M, N, K, W8A8_ACT_NONE,
                            workspace, ws_bytes, stream);
}

const char *w8a8_gemm_kernel_name(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1) return "invalid";
  if (use_decode_path(M)) return "decode_kernel (swap-AB stream-K, needs a workspace)";
  switch (choose_large(M, N)) {
    case LargeKind::kPair: return "gemm2sm_kernel<256, 3> (2-SM pair, 256x256 tiles)";
    case LargeKind::kPair128: return "gemm2sm_kernel<128, 4> (2-SM pair, 256x128 tiles)";
    case LargeKind::k256: return "gemm_kernel<256, 4, 1> (1-SM, 128x256 tiles)";
    default: return "gemm_kernel<128, 3, 2> (1-SM, 128x128 tiles, 2 k-blocks per stage)";
  }
}

w8a8_status w8a8_scaled_mm_i32(const int8_t *q, const void *packed_w, int32_t *acc, int64_t M,
                               int64_t N, int64_t K, w8a8_stream_t stream) {
  w8a8_status st = check_gemm_args(q, packed_w, acc, M, N, K);
  if (st != W8A8_OK) return st;
  return launch_scaled_mm(q, nullptr, packed_w, nullptr, nullptr, acc, true, M, N, K,
                          reinterpret_cast<cudaStream_t>(stream), false);
}

w8a8_status w8a8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, size_t *bytes) {
  if (!bytes || M < 1 || N < 1 || K < 1) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0) return W8A8_ERR_UNSUPPORTED_SHAPE;
  *bytes = (size_t)linear_workspace_bytes(M, N, K);
  return W8A8_OK;
}

w8a8_status w8a8_linear_act(const void *x, int64_t ldx, const void *packed_w,
                            const float *w_scale, const void *bias, void *y, int64_t M, int64_t N,
                            int64_t K, int act, void *workspace, size_t ws_bytes,
                            w8a8_stream_t stream) {
  w8a8_status st = check_gemm_args(x, packed_w, y, M, N, K);
  if (st != W8A8_OK) return st;
  if (!w_scale || !workspace) return W8A8_ERR_INVALID_ARG;
  if (ldx < K) return W8A8_ERR_INVALID_ARG;
  if (act != W8A8_ACT_NONE && act != W8A8_ACT_GELU_TANH) return W8A8_ERR_INVALID_ARG;
  if (ldx % 8 != 0 || !aligned16(w_scale) || !aligned16(workspace) ||
      (bias && !aligned16(bias)))
    return W8A8_ERR_ALIGNMENT;
  if ((int64_t)ws_bytes < linear_workspace_bytes(M, N, K)) return W8A8_ERR_BUFFER_TOO_SMALL;
  if (!use_decode_path(M) && forced_path() == 2) return W8A8_ERR_INVALID_ARG;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int8_t *q = reinterpret_cast<int8_t *>(ws);
  float *a_scale = reinterpret_cast<float *>(ws + round_up(M * K, 256));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  st = launch_quant(x, M, K, ldx, q, a_scale, s, true);
  if (st != W8A8_OK) return st;
  if (use_decode_path(M)) {
    void *dws = ws + round_up(M * K, 256) + round_up(M * 4, 256);
    return launch_decode(q, a_scale, packed_w, w_scale, bias, y, M, N, K, dws, s, true, act);
  }
  return launch_scaled_mm(q, a_scale, packed_w, w_scale, bias, y, false, M, N, K, s, true, act,
                          true);
}

w8a8_status w8a8_linear(const void *x, int64_t ldx, const void *packed_w, const float *w_scale,
                        const void *bias, void *y, int64_t M, int64_t N, int64_t K,
                        void *workspace, size_t ws_bytes, w8a8_stream_t stream) {
  return w8a8_linear_act(x, ldx, packed_w, w_scale, bias, y, M, N, K, W8A8_ACT_NONE, workspace,
                         ws_bytes, stream);
}

w8a8_status w8a8_linear_act_quant_workspace_bytes(int64_t M, int64_t N, int64_t K,
                                                  size_t *bytes) {
  if (!bytes || M < 1 || N < 1 || K < 1) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0) return W8A8_ERR_UNSUPPORTED_SHAPE;
  *bytes = (size_t)act_quant_workspace_bytes(M, N, K);
  return W8A8_OK;
}

w8a8_status w8a8_linear_act_quant(const void *x, int64_t ldx, const void *packed_w,
                                  const float *w_scale, const void *bias, void *y, int64_t M,
                                  int64_t N, int64_t K, int act, int8_t *q_next,
                                  float *a_scale_next, void *workspace, size_t ws_bytes,
                                  w8a8_stream_t stream) {
  w8a8_status st = check_gemm_args(x, packed_w, y, M, N, K);
  if (st != W8A8_OK) return st;
  if (!w_scale || !workspace || !q_next || !a_scale_next) return W8A8_ERR_INVALID_ARG;
  if (ldx < K) return W8A8_ERR_INVALID_ARG;
  if (act != W8A8_ACT_NONE && act != W8A8_ACT_GELU_TANH) return W8A8_ERR_INVALID_ARG;
  // the codes are the next layer's GEMM input, K = N; the codes' work units
  // (rows x 2048 columns) are counted in 32 bits
  if (N > kMaxFusedN || N % 16 != 0 || M * ((N + 2047) / 2048) >= ((int64_t)1 << 31))
    return W8A8_ERR_UNSUPPORTED_SHAPE;
  if (ldx % 8 != 0 || !aligned16(w_scale) || !aligned16(workspace) ||
      (bias && !aligned16(bias)) || !aligned16(q_next) || !aligned16(a_scale_next))
    return W8A8_ERR_ALIGNMENT;
  if ((int64_t)ws_bytes < act_quant_workspace_bytes(M, N, K)) return W8A8_ERR_BUFFER_TOO_SMALL;
  if (!use_decode_path(M) && forced_path() == 2) return W8A8_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (use_decode_path(M)) {
    // Few rows: the layer, then the quantisation of its output.
    st = w8a8_linear_act(x, ldx, packed_w, w_scale, bias, y, M, N, K, act, workspace, ws_bytes,
                         stream);
    if (st != W8A8_OK) return st;
    return launch_quant(y, M, N, N, q_next, a_scale_next, s, false);
  }
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int8_t *q = reinterpret_cast<int8_t *>(ws);
  int64_t off = round_up(M * K, 256);
  float *a_scale = reinterpret_cast<float *>(ws + off);
  off += round_up(M * 4, 256);
  uint32_t *row_amax = reinterpret_cast<uint32_t *>(ws + off);
  off += round_up(M * 4, 256);
  unsigned long long *row_done = reinterpret_cast<unsigned long long *>(ws + off);
  off += round_up(((M + 127) / 128) * 8, 256);
  unsigned long long *exit_word = reinterpret_cast<unsigned long long *>(ws + off);
  RowSignal sig{row_amax, row_done, next_call_tag() & 0xFFFFFFFFull, q_next, a_scale_next,
                exit_word};
  if (sig.tag == 0) sig.tag = 1;
  st = launch_quant(x, M, K, ldx, q, a_scale, s, true, row_amax);
  if (st != W8A8_OK) return st;
  return launch_scaled_mm(q, a_scale, packed_w, w_scale, bias, y, false, M, N, K, s, true, act,
                          true, &sig);
}

}  // extern "C"
