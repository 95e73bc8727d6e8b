// gemm2sm.cu -- int8 GEMM + dequantising epilogue with 2-SM tensor-core MMAs.
//
// Same arithmetic as gemm.cu ("Issue 5 probe: int8 quantized DiT serve paths
// on the RTX 3090", Round two: int8 scaled matmul with per-token and
// per-channel fp32 scales; "INT8 Quant for Dual-Max Recipe": native int8 x int8
// on the tensor cores), organised for CTA pairs:
//
//   * output tiles are 256 x 256; the even CTA of a pair owns rows 0..127 of
//     the tile, the odd CTA rows 128..255.  Each CTA loads only its own 128
//     rows of q and its own 128-row slab of the packed weights (the tile's N
//     half), so per SM a k-block moves 32 KB for 128 x 256 x 128 MACs -- two
//     thirds of what a 1-SM 128 x 256 tile moves;
//   * a pipeline stage holds two k-blocks (64 KB per CTA), fetched with three
//     TMA copies (two q boxes, one 32 KB box of two contiguous packed weight
//     tiles), all completing on the even CTA's "full" barrier;
//   * the even CTA's elected thread issues tcgen05.mma.cta_group::2.kind::i8
//     (M = 256, N = 256, K = 32), which reads both CTAs' shared memory and
//     accumulates into both CTAs' TMEM; its commits arrive on the "empty" and
//     "accumulator full" barriers of both CTAs (commit multicast);
//   * both CTAs run the epilogue on their own 128 TMEM lanes;
//   * roles and limits as in gemm.cu: the producer is the lone thread of a
//     last, one-thread warp and walks its (segment, stage) list with a cursor;
//     at most 128 registers a thread.
//
// Persistent clusters of 2 CTAs, double-buffered accumulators.  When the
// 256 x 256 tiles fill the SM pairs a few times over plus a short last round
// (at most half the pairs), the tiles of that round run as their two
// 256 x 128 halves instead (MMA N = 128, each CTA loading 64 weight rows),
// spread over twice as many pairs.
//
// No TMA load uses cluster multicast.  Every wait is time-bounded (the waits
// between the two CTAs of a pair are safe: a cluster's CTAs are
// co-scheduled); a block that gives up drains its copies, the cluster meets
// at a barrier and frees TMEM.
#include <algorithm>

#include "gemm_common.cuh"

namespace w8a8 {
namespace {

constexpr int kStageK = 2;                        // k-blocks per stage
constexpr int kHalfStage = kStageK * kTileBytes;  // 32 KB: the q part of one stage

// BN = tile N of the pair (256 or 128); each CTA holds BN/2 weight rows.
template <int BN, int STAGES>
struct PairSmem {
  static constexpr int kBRows = BN / 2;                 // weight rows per CTA
  static constexpr int kBTile = kBRows * kBK;           // weight bytes per k-block per CTA
  static constexpr int kBStage = kStageK * kBTile;
  static constexpr int kA = 0;                          // STAGES x 32 KB q tiles
  static constexpr int kB = STAGES * kHalfStage;        // STAGES x kBStage weight tiles
  static constexpr int kEpiPerWarp = (BN / 2) * 6;  // BN/2 columns: fp32 scale + bf16 bias
  static constexpr int kEpi = kB + STAGES * kBStage;
  static constexpr int kEpiEnd = kEpi + kEpiWarps * kEpiPerWarp;
  static constexpr int kOut = kEpiEnd + 1024 - kEpiEnd % 1024;
  // full[S], empty[S], tfull[2], tempty[2], done
  static constexpr int kBars = kOut + kEpiWarps * kEpiStagePerWarp;
  static constexpr int kMisc = kBars + (2 * STAGES + 5) * 8;
  static constexpr int kUsed = kMisc + 16;
  static constexpr int kAlloc = kUsed + 1024;
};

// At most kGemmRegs registers a thread, so that a CTA (11 warps) fits on an
// SM beside the blocks of the quantisation kernel it is launched behind and
// starts its prologue and first weight copies while they run.
// ROWMAX: the next layer's quantisation is fused in (GemmArgs::row_amax).
template <int BN, int STAGES, bool ROWMAX>
__global__ void __maxnreg__(kGemmRegs)
    gemm2sm_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_w,
                   const __grid_constant__ CUtensorMap tmap_w64,
                   const __grid_constant__ CUtensorMap tmap_y, const GemmArgs args) {
  using L = PairSmem<BN, STAGES>;
  constexpr int kPairBN = BN;
  constexpr uint32_t kTmemCols = 2 * BN;
  constexpr uint32_t kIdesc = idesc_i8(256, BN);
  constexpr uint32_t kIdescHalf = idesc_i8(256, 128);  // a 256 x 128 half of a 256-wide tile
  constexpr int kHalfBTile = 64 * kBK;                   // its weight rows per CTA per k-block

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
  const uint32_t crank = cluster_ctarank();
  const uint32_t rank = crank & 1;      // 0: even CTA of the pair (issues the MMAs)
  const uint32_t lead = crank & ~1u;    // cluster rank of this pair's even CTA
  // commit multicast masks are in cluster-rank space
  const uint16_t pair_mask = (uint16_t)(0x3u << lead);
  const uint16_t self_mask = (uint16_t)(0x1u << crank);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);  // one expect_tx arrival from each CTA of the pair
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 2 * kEpiWarps);  // the epilogue warps of both CTAs
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_w);
    if (BN == 256 && args.full_tiles < args.tiles_m * args.tiles_n) prefetch_tmap(&tmap_w64);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of the cluster initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = args.tiles_m * args.tiles_n;  // 256 x BN tiles
  const int num_kb = args.num_kb;
  const int S = (num_kb + kStageK - 1) / kStageK;  // stages per tile
  const int slot = (int)(blockIdx.x >> 1);
  const int nslots = (int)(gridDim.x >> 1);
  // Work items: tiles [0, full_tiles) whole, then item full_tiles + 2 j + h
  // is N half h of tile full_tiles + j.  This pair takes items slot,
  // slot + nslots, ... (one segment of S stages each).
  const int num_items = args.full_tiles + 2 * (num_tiles - args.full_tiles);
  auto item_tile = [&](int item) -> int {
    return item < args.full_tiles ? item : args.full_tiles + ((item - args.full_tiles) >> 1);
  };
  auto item_half = [&](int item) -> int {  // -1: the whole tile
    return item < args.full_tiles ? -1 : ((item - args.full_tiles) & 1);
  };
  const int nseg = slot < num_items ? (num_items - 1 - slot) / nslots + 1 : 0;
  auto seg_tile = [&](int i) -> int { return slot + i * nslots; };
  const uint32_t my_iters = (uint32_t)nseg * (uint32_t)S;
  const uint32_t full0 = map_to_cta(smem_addr(full), lead);  // pair leader's full[0]
  const uint32_t tempty0 = map_to_cta(smem_addr(tempty), lead);

  // Roles (as in the 1-SM kernel): the producer is the lone thread of a last,
  // one-thread warp, so no parked lane of its warp slows its wait-then-copy
  // loop (fused QKV 28.7 -> 28.0 us); lane 0 of warp 1 issues the MMAs; warp
  // 0 is idle.
  if (threadIdx.x == kGemmThreads) {
    // ---------------- producer (every CTA) ----------------
    // A cursor walks this CTA's (segment, stage) list in the order the MMAs
    // consume it.  A segment's box coordinates (divisions by the runtime tile
    // counts) are formed when the cursor enters it, after the previous
    // stage's copies are issued, so a released slot is refilled with the
    // copies alone (the issuing thread is on the ring's critical path).
    struct Cursor {
      int seg, st;  // segment index, stage within the tile
      int kind;     // 0: 256 x BN tile, 1: 256 x 128 half of a 256-wide tile
      int wrow;     // weight box row of k-block 0 (plus 128 per k-block)
      int qrow;     // first q row of this CTA
    };
    auto enter = [&](int i, int st) {
      Cursor c;
      c.seg = i;
      c.st = st;
      if (i >= nseg) {
        c.kind = 0;
        c.wrow = c.qrow = 0;
        return c;
      }
      const int item = seg_tile(i), tile = item_tile(item), half = item_half(item);
      int mb, nb;
      tile_coords<ROWMAX>(args, tile, mb, nb);
      c.kind = (BN == 256 && half >= 0) ? 1 : 0;
      c.qrow = mb * 256 + (int)rank * 128;
      if (BN == 256 && half >= 0)
        c.wrow = (nb * 2 + half) * num_kb * 128 + (int)rank * 64;  // this CTA's 64 rows
      else if (BN == 256)
        c.wrow = (nb * 2 + (int)rank) * num_kb * 128;  // this CTA's 128-row slab
      else
        c.wrow = nb * num_kb * 128 + (int)rank * 64;  // this CTA's 64 rows of slab nb
      return c;
    };
    auto advance = [&](Cursor &c) {
      if (++c.st >= S) c = enter(c.seg + 1, 0);
    };
    auto stage_nk = [&](const Cursor &c) { return min(kStageK, num_kb - c.st * kStageK); };
    auto stage_bytes = [&](const Cursor &c, int nk) {
      // the 256-wide weight box always moves two tiles (zero-filled past the end)
      const int wb = BN == 256 ? (c.kind == 1 ? nk * kHalfBTile : L::kBStage) : nk * L::kBTile;
      return (uint32_t)(nk * kTileBytes + wb);
    };
    auto weights = [&](const Cursor &c, uint32_t s, int nk) {
      const uint32_t bar = full0 + s * 8;
      const int row = c.wrow + c.st * kStageK * 128;
      if (BN == 256 && c.kind == 0) {
        // two contiguous packed tiles (k-blocks kb0, kb0+1) of this CTA's slab
        tma_load_2d_pair(sB + s * L::kBStage, &tmap_w, 0, row, bar);
      } else {
        const int step = (BN == 256) ? kHalfBTile : L::kBTile;
        for (int h = 0; h < nk; ++h)
          tma_load_2d_pair(sB + s * L::kBStage + h * step, BN == 256 ? &tmap_w64 : &tmap_w, 0,
                           row + h * 128, bar);
      }
    };
    auto acts = [&](const Cursor &c, uint32_t s, int nk) {
      const uint32_t bar = full0 + s * 8;
      for (int h = 0; h < nk; ++h)
        tma_load_2d_pair(sA + s * kHalfStage + h * kTileBytes, &tmap_q, (c.st * kStageK + h) * kBK,
                         c.qrow, bar);
    };
    const uint32_t pre = my_iters < (uint32_t)STAGES ? my_iters : (uint32_t)STAGES;
    uint32_t issued = 0;
    bool ok = true;
    if (my_iters > 0) {
      Cursor cur = enter(0, 0);
      const Cursor first = cur;
      // weight tiles do not depend on the preceding kernel: issue them first
      for (uint32_t it = 0; it < pre; ++it) {
        const int nk = stage_nk(cur);
        mbar_arrive_expect_tx_cluster(full0 + it * 8, stage_bytes(cur, nk));
        weights(cur, it, nk);
        advance(cur);
      }
      griddep_wait();
      {
        Cursor c = first;
        for (uint32_t it = 0; it < pre; ++it) {
          acts(c, it, stage_nk(c));
          advance(c);
        }
      }
      uint32_t s = 0, ph = 1;  // stage `pre` (if any) reuses slot 0, second round
      for (issued = pre; issued < my_iters; ++issued) {
        const int nk = stage_nk(cur);
        const uint32_t bytes = stage_bytes(cur, nk);
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx_cluster(full0 + s * 8, bytes);
        weights(cur, s, nk);
        acts(cur, s, nk);
        advance(cur);
        if (++s == (uint32_t)STAGES) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    // Wait until every stage this CTA filled has been consumed: the MMA
    // commits that release them also arrive here, and must land before the
    // CTA may leave.  The last stage issued into slot sl has parity
    // (last / STAGES) & 1.
    if (ok)
      for (uint32_t sl = 0; sl < (uint32_t)STAGES && sl < issued; ++sl) {
        const uint32_t last = sl + ((issued - 1 - sl) / STAGES) * STAGES;
        volatile int no_abort = 0;
        (void)mbar_wait_bounded(&empty[sl], (last / STAGES) & 1, &no_abort, args.status);
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
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (even CTA of each pair) ----------------
      // Slot, phase and operand descriptors advance by counters (a
      // descriptor's address field is the shared-memory address / 16).
      const uint64_t a_desc0 = sw128_kmajor_desc(sA), b_desc0 = sw128_kmajor_desc(sB);
      uint32_t s = 0, ph = 0;
      bool ok = true;
      for (int i = 0; ok && i < nseg; ++i) {
        const uint32_t b = i & 1, bph = (i >> 1) & 1;
        if (!mbar_wait(&tempty[b], bph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kPairBN;
        const bool half = BN == 256 && item_half(seg_tile(i)) >= 0;
        const uint32_t idesc = half ? kIdescHalf : kIdesc;
        const int b_step = half ? kHalfBTile : L::kBTile;
        for (int st = 0; st < S; ++st) {
          const int nk = min(kStageK, num_kb - st * kStageK);
          const uint64_t a_desc = a_desc0 + ((s * kHalfStage) >> 4);
          const uint64_t b_desc = b_desc0 + ((s * L::kBStage) >> 4);
          if (!mbar_wait(&full[s], ph, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int h = 0; h < nk; ++h) {
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_i8_pair(d_tmem, a_desc + ((h * kTileBytes) >> 4) + 2 * k,
                          b_desc + ((h * b_step) >> 4) + 2 * k, idesc,
                          st != 0 || h != 0 || k != 0);
          }
          mma_commit_pair(&empty[s], pair_mask);  // frees the stage in both CTAs
          if (++s == (uint32_t)STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) mma_commit_pair(&tfull[b], pair_mask);
      }
      if (!ok) {
        mma_commit_pair(mma_done, self_mask);
        volatile int no_abort = 0;
        (void)mbar_wait_bounded(mma_done, 0, &no_abort, args.status);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9, every CTA) ----------------
    griddep_wait();  // a_scale comes from the preceding kernel
    constexpr int kCols = kPairBN / 2;  // columns of the tile this warp drains
    const EpiWarp ew(warp);
    float *s_ws = reinterpret_cast<float *>(smem + L::kEpi + (warp - 2) * L::kEpiPerWarp);
    uint16_t *s_bias = reinterpret_cast<uint16_t *>(s_ws + kCols);
    uint8_t *s_out = smem + L::kOut + (warp - 2) * kEpiStagePerWarp;
    const int j0 = ew.half * kCols;  // first tile column of this warp
    CodesCursor cursor = codes_cursor(args, warp - 1);  // (ROWMAX) this warp's codes units
    for (int i = 0; i < nseg; ++i) {
      const int tile = item_tile(seg_tile(i)), half = item_half(seg_tile(i));
      int mb, nb;
      tile_coords<ROWMAX>(args, tile, mb, nb);
      const int row0 = mb * 256 + (int)rank * 128 + ew.quarter * 32;
      // a half tile's 128 columns: 64 per warp
      const int jw = half >= 0 ? half * 128 + ew.half * 64 : j0;  // warp's first tile column
      const int ncols = half >= 0 ? 64 : kCols;
      const int n0 = nb * kPairBN + jw;
      const uint32_t b = i & 1, bph = (i >> 1) & 1;
      stage_columns<kCols>(args, n0, lane, s_ws, s_bias);
      const float as = row0 + lane < args.M ? __ldg(args.a_scale + row0 + lane) : 0.0f;
      __syncwarp();
      if (ROWMAX) codes_while_waiting(args, lane, cursor, &tfull[b], bph);
      int ok = 0;
      if (lane == 0) ok = mbar_wait(&tfull[b], bph, abort_flag, args.status);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + b * kPairBN + (half >= 0 ? ew.half * 64 : j0) +
                             ((uint32_t)(ew.quarter * 32) << 16);
      // dequantise: acc * a_scale * w_scale + bias
      uint32_t rmax = 0;
      epilogue_tma<kCols, ROWMAX>(args, &tmap_y, taddr, lane, row0, n0, as, s_ws, s_bias, s_out,
                                  rmax, ncols);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + b * 8);
      // (the odd CTA of the last row tile may hold rows wholly past M)
      if (ROWMAX && n0 < args.N && (row0 >> 7) * 128 < args.M)
        publish_rows(args, lane, row0, row_max_bits(rmax), min(ncols, args.N - n0));
    }
    if (lane == 0) bulk_wait_group_all();  // output stores complete before exit
    __syncwarp();
    if (ROWMAX)  // help with the codes still to form
      while (codes_next(args, lane, cursor, true, abort_flag)) {
      }
  }

  tc_fence_before();
  cluster_sync();  // no CTA leaves while a peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  if (ROWMAX) codes_exit(args);
}

FuncAttrOnce g_pair_smem_attr[4];  // one per kernel instance (`slot_id`)

template <int BN, int STAGES, bool ROWMAX = false>
w8a8_status run_pair(const CUtensorMap &tq, const CUtensorMap &tw, const CUtensorMap &tw64,
                     const CUtensorMap &ty, const GemmArgs &a, cudaStream_t stream, bool pdl,
                     int slot_id) {
  using L = PairSmem<BN, STAGES>;
  auto k = gemm2sm_kernel<BN, STAGES, ROWMAX>;
  if (g_pair_smem_attr[slot_id].ensure([&] {
        return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
      }) != cudaSuccess)
    return W8A8_ERR_CUDA;
  const int tiles = a.tiles_m * a.tiles_n;
  const int items = a.full_tiles + 2 * (tiles - a.full_tiles);
  // persistent: one pair per two SMs, at most one per work item
  const int pairs = std::max(1, std::min(items, sm_count() / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kGemmThreads + 1);  // + the producer's one-thread warp
  cfg.dynamicSmemBytes = (size_t)L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, tq, tw, tw64, ty, a);
  count_launch();
  return from_cuda(e);
}

}  // namespace

// Number of 256 x bn tiles the pair kernel would process.
int64_t pair_tiles(int64_t M, int64_t N, int bn) { return ((M + 255) / 256) * ((N + bn - 1) / bn); }

// Whole 256 x 256 tiles before the ones that run as two 256 x 128 halves:
// when the tiles fill the SM pairs more than once and leave a last round of
// at most half the pairs, that round's tiles are split (twice as many items,
// each about 3/4 of a tile's time: the halves move 3/4 of the bytes).
int64_t pair_full_tiles(int64_t tiles, int64_t pairs) {
  const int64_t rem = tiles % pairs;
  return (tiles > pairs && rem > 0 && 2 * rem <= pairs) ? tiles - rem : tiles;
}

w8a8_status launch_gemm2sm(const int8_t *q, const float *a_scale, const void *packed_w,
                           const float *w_scale, const void *bias, void *y, int64_t M, int64_t N,
                           int64_t K, cudaStream_t stream, bool pdl, int bn, int act,
                           const RowSignal *sig) {
  CUtensorMap tq, tw, tw64, ty;
  if (!make_tmap_u8_2d(&tq, q, (uint64_t)M, (uint64_t)K, (uint64_t)K, kBM, kBK))
    return W8A8_ERR_CUDA;
  if (!make_tmap_out_bf16(&ty, y, (uint64_t)M, (uint64_t)N)) return W8A8_ERR_CUDA;
  const uint64_t wrows = (uint64_t)(packed_rows(N) * packed_cols(K) / 128);
  if (!make_tmap_u8_2d_plain(&tw, packed_w, wrows, 128, 128, bn == 128 ? 64 : 256, 128))
    return W8A8_ERR_CUDA;
  if (!make_tmap_u8_2d_plain(&tw64, packed_w, wrows, 128, 128, 64, 128)) return W8A8_ERR_CUDA;
  GemmArgs a{};
  a.packed_w = static_cast<const uint8_t *>(packed_w);
  a.a_scale = a_scale;
  a.w_scale = w_scale;
  a.bias = static_cast<const uint16_t *>(bias);
  a.out = y;
  a.M = (int)M;
  a.N = (int)N;
  a.num_kb = (int)(packed_cols(K) / 128);
  a.tiles_m = (int)((M + 255) / 256);
  a.tiles_n = (int)((N + bn - 1) / bn);
  a.full_tiles = a.tiles_m * a.tiles_n;
  // Re-read the smaller operand wave after wave: with M > N the weights
  // (DiT MLP down-projection, 4096 x 3072 x 12288: q read from DRAM 151 MB
  // a launch in column-tile order, for 88 MB of operands; GEMM 2 % faster).
  a.row_major = M > N ? 1 : 0;
  a.act = act;
  a.status = status_word();
  if (!a.status) return W8A8_ERR_CUDA;
  if (sig) {
    a.row_amax = sig->row_amax;
    a.row_done = sig->row_done;
    a.done_tag = sig->tag;
    a.q_next = sig->q_next;
    a.a_scale_next = sig->a_scale_next;
    a.exit_word = sig->exit_word;
  }
  if (bn == 128)
    return sig ? run_pair<128, 4, true>(tq, tw, tw64, ty, a, stream, pdl, 3)
               : run_pair<128, 4>(tq, tw, tw64, ty, a, stream, pdl, 1);
  a.full_tiles = (int)pair_full_tiles(a.full_tiles, sm_count() / 2);
  return sig ? run_pair<256, 3, true>(tq, tw, tw64, ty, a, stream, pdl, 2)
             : run_pair<256, 3>(tq, tw, tw64, ty, a, stream, pdl, 0);
}

}  // namespace w8a8
