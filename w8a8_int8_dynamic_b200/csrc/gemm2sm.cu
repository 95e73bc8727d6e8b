// gemm2sm.cu -- int8 GEMM + dequantising epilogue with 2-SM tensor-core MMAs.
//
// Same arithmetic as gemm.cu ("Issue 5 probe: int8 quantized DiT serve paths
// on the RTX 3090", Round two: int8 scaled matmul with per-token and
// per-channel fp32 scales; "INT8 Quant for Dual-Max Recipe": native int8 x int8
// on the tensor cores), organised for a CTA pair (a 2-CTA cluster):
//
//   * output tiles are 256 x 256; the even CTA owns rows 0..127 of the tile,
//     the odd CTA rows 128..255.  Each CTA loads only its own 128 rows of q
//     and its own 128-row slab of the packed weights (the tile's N half), so
//     per SM a k-block moves 32 KB for 128 x 256 x 128 MACs -- two thirds of
//     what a 1-SM 128 x 256 tile moves, which is what lets the tensor pipe be
//     fed from L2 at the int8 rate;
//   * a pipeline stage holds two k-blocks (64 KB per CTA), fetched with three
//     TMA copies (two q boxes, one 32 KB box of two contiguous packed weight
//     tiles), all completing on the even CTA's "full" barrier;
//   * the even CTA's elected thread issues tcgen05.mma.cta_group::2.kind::i8
//     (M = 256, N = 256, K = 32), which reads both CTAs' shared memory and
//     accumulates into both CTAs' TMEM; its commits arrive on the "empty" and
//     "accumulator full" barriers of both CTAs (commit multicast);
//   * both CTAs run the epilogue on their own 128 TMEM lanes and tell the
//     even CTA when an accumulator buffer may be reused.
//
// No TMA load uses cluster multicast.  Every wait is time-bounded; a block
// that gives up drains its copies, the pair meets at a cluster barrier and
// frees TMEM.
#include <algorithm>

#include "gemm_common.cuh"

namespace w8a8 {
namespace {

constexpr int kPairBN = 256;                 // tile N (both CTAs)
constexpr int kStageK = 2;                   // k-blocks per stage
constexpr int kHalfStage = kStageK * kTileBytes;  // 32 KB: one operand of one stage

template <int STAGES>
struct PairSmem {
  static constexpr int kA = 0;                          // STAGES x 32 KB q tiles
  static constexpr int kB = STAGES * kHalfStage;        // STAGES x 32 KB weight tiles
  static constexpr int kEpiPerWarp = kPairBN * 4 + kPairBN * 2;
  static constexpr int kEpi = kB + STAGES * kHalfStage;
  static constexpr int kBars = kEpi + 4 * kEpiPerWarp;  // full, empty, tfull[2], tempty[2], done
  static constexpr int kMisc = kBars + (2 * STAGES + 5) * 8;
  static constexpr int kUsed = kMisc + 16;
  static constexpr int kAlloc = kUsed + 1024;
};

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    gemm2sm_kernel(const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_w, const GemmArgs args) {
  using L = PairSmem<STAGES>;
  constexpr uint32_t kTmemCols = 2 * kPairBN;
  constexpr uint32_t kIdesc = idesc_i8(256, kPairBN);

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

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: even CTA (issues the MMAs), 1: odd CTA
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 2);  // one expect_tx arrival from each CTA of the pair
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);  // four epilogue warps in each CTA
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_w);
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, kTmemCols);
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = args.tiles_m * args.tiles_n;  // 256 x 256 tiles
  const int num_kb = args.num_kb;
  const int num_stages_k = (num_kb + kStageK - 1) / kStageK;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int my_tiles = pair < num_tiles ? (num_tiles - 1 - pair) / npairs + 1 : 0;
  const uint32_t my_iters = (uint32_t)my_tiles * num_stages_k;
  const uint32_t full0 = map_to_cta(smem_addr(full), 0);  // even CTA's full[0]
  const uint32_t tempty0 = map_to_cta(smem_addr(tempty), 0);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer (both CTAs) ----------------
      auto tile_of = [&](uint32_t it) { return pair + (int)(it / num_stages_k) * npairs; };
      auto issue = [&](uint32_t it, uint32_t s, bool weights, bool acts) {
        const int tile = tile_of(it);
        const int mb = tile % args.tiles_m, nb = tile / args.tiles_m;
        const int kb0 = (int)(it % num_stages_k) * kStageK;
        const int nk = min(kStageK, num_kb - kb0);
        const uint32_t bar = full0 + s * 8;
        if (weights) {
          // two contiguous packed tiles (k-blocks kb0, kb0+1) of this CTA's slab
          const int slab = nb * 2 + (int)rank;
          tma_load_2d_pair(sB + s * kHalfStage, &tmap_w, 0, (slab * num_kb + kb0) * 128, bar);
        }
        if (acts) {
          const int row0 = mb * 256 + (int)rank * 128;
          for (int h = 0; h < nk; ++h)
            tma_load_2d_pair(sA + s * kHalfStage + h * kTileBytes, &tmap_q, (kb0 + h) * kBK, row0,
                             bar);
        }
      };
      auto stage_bytes = [&](uint32_t it) {
        const int kb0 = (int)(it % num_stages_k) * kStageK;
        return (uint32_t)(kHalfStage + min(kStageK, num_kb - kb0) * kTileBytes);
      };
      uint32_t last_par[STAGES];
      bool ok = true;
      const uint32_t pre = my_iters < (uint32_t)STAGES ? my_iters : (uint32_t)STAGES;
      // weight tiles do not depend on the preceding kernel: issue them first
      for (uint32_t it = 0; it < pre; ++it) {
        mbar_arrive_expect_tx_cluster(full0 + it * 8, stage_bytes(it));
        issue(it, it, true, false);
        last_par[it] = 0;
      }
      griddep_wait();
      for (uint32_t it = 0; it < pre; ++it) issue(it, it, false, true);
      for (uint32_t it = pre; it < my_iters; ++it) {
        const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx_cluster(full0 + s * 8, stage_bytes(it));
        issue(it, s, true, true);
        last_par[s] = ph;
      }
      // Wait until every stage this CTA filled has been consumed: the MMA
      // commits that release them also arrive here, and must land before the
      // pair may leave.  On abort, wait for our own copies instead.
      for (uint32_t s = 0; s < (uint32_t)STAGES && s < my_iters; ++s) {
        volatile int no_abort = 0;
        if (ok)
          (void)mbar_wait_bounded(&empty[s], last_par[s], &no_abort, args.status);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (even CTA) ----------------
      uint32_t it = 0;
      bool ok = true;
      for (int t = 0; ok && t < my_tiles; ++t) {
        const uint32_t b = t & 1, bph = (t >> 1) & 1;
        if (!mbar_wait(&tempty[b], bph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kPairBN;
        for (int j = 0; j < num_stages_k; ++j, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(kStageK, num_kb - j * kStageK);
          for (int h = 0; h < nk; ++h) {
            const uint64_t a_desc = sw128_kmajor_desc(sA + s * kHalfStage + h * kTileBytes);
            const uint64_t b_desc = sw128_kmajor_desc(sB + s * kHalfStage + h * kTileBytes);
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_i8_pair(d_tmem, a_desc + 2 * k, b_desc + 2 * k, kIdesc, (j | h | k) != 0);
          }
          mma_commit_pair(&empty[s], 0x3);  // frees the stage in both CTAs
        }
        if (ok) mma_commit_pair(&tfull[b], 0x3);
      }
      if (!ok) {
        mma_commit_pair(mma_done, 0x1);
        volatile int no_abort = 0;
        (void)mbar_wait_bounded(mma_done, 0, &no_abort, args.status);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5, both CTAs) ----------------
    griddep_wait();  // a_scale comes from the preceding kernel
    const int quarter = warp & 3;
    float *s_ws = reinterpret_cast<float *>(smem + L::kEpi + (warp - 2) * L::kEpiPerWarp);
    uint16_t *s_bias = reinterpret_cast<uint16_t *>(s_ws + kPairBN);
    for (int t = 0; t < my_tiles; ++t) {
      const int tile = pair + t * npairs;
      const int mb = tile % args.tiles_m, nb = tile / args.tiles_m;
      const int row_base = mb * 256 + (int)rank * 128;
      const uint32_t b = t & 1, bph = (t >> 1) & 1;
      stage_columns<kPairBN>(args, nb, lane, s_ws, s_bias);
      const int row = row_base + quarter * 32 + lane;
      const float as = row < args.M ? __ldg(args.a_scale + row) : 0.0f;
      __syncwarp();
      int ok = 0;
      if (lane == 0) ok = mbar_wait(&tfull[b], bph, abort_flag, args.status);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      epilogue_tile<kPairBN, false>(args, tmem_base + b * kPairBN, quarter, lane, row_base, nb, as,
                                    s_ws, s_bias);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + b * 8);
    }
  }

  tc_fence_before();
  cluster_sync();  // no CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

constexpr int kPairStages = 3;
bool g_pair_attr_done[64];

}  // namespace

// Number of 256 x 256 tiles the pair kernel would process.
int64_t pair_tiles(int64_t M, int64_t N) { return ((M + 255) / 256) * ((N + 255) / 256); }

w8a8_status launch_gemm2sm(const int8_t *q, const float *a_scale, const void *packed_w,
                           const float *w_scale, const void *bias, void *y, int64_t M, int64_t N,
                           int64_t K, cudaStream_t stream, bool pdl) {
  CUtensorMap tq, tw;
  if (!make_tmap_u8_2d(&tq, q, (uint64_t)M, (uint64_t)K, (uint64_t)K, kBM, kBK))
    return W8A8_ERR_CUDA;
  const uint64_t wrows = (uint64_t)(packed_rows(N) * packed_cols(K) / 128);
  if (!make_tmap_u8_2d_plain(&tw, packed_w, wrows, 128, 128, 256, 128)) return W8A8_ERR_CUDA;
  GemmArgs a;
  a.packed_w = static_cast<const uint8_t *>(packed_w);
  a.a_scale = a_scale;
  a.w_scale = w_scale;
  a.bias = static_cast<const uint16_t *>(bias);
  a.out = y;
  a.M = (int)M;
  a.N = (int)N;
  a.num_kb = (int)(packed_cols(K) / 128);
  a.tiles_m = (int)((M + 255) / 256);
  a.tiles_n = (int)((N + 255) / 256);
  a.status = status_word();
  if (!a.status) return W8A8_ERR_CUDA;
  using L = PairSmem<kPairStages>;
  auto k = gemm2sm_kernel<kPairStages>;
  const int d = current_device();
  if (d < 0 || d >= 64 || !g_pair_attr_done[d]) {
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
        cudaSuccess)
      return W8A8_ERR_CUDA;
    if (d >= 0 && d < 64) g_pair_attr_done[d] = true;
  }
  const int tiles = a.tiles_m * a.tiles_n;
  const int pairs = std::max(1, std::min(tiles, sm_count() / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs));
  cfg.blockDim = dim3(kThreads);
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, k, tq, tw, a);
  count_launch();
  return from_cuda(e);
}

}  // namespace w8a8
