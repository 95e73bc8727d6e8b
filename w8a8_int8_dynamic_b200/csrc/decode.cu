// decode.cu -- small-M (decode) W8A8 GEMM that streams the weights at HBM rate.
//
// Source: "INT8 Quant for Dual-Max Recipe (To replace the FP8 one)": decode is
// memory-bandwidth-bound -- an 8-bit weight moves the same bytes per token
// whatever the format, so the weight stream sets the speed; "Issue 5 probe:
// int8 quantized DiT serve paths on the RTX 3090", Round two: the same int8
// scaled matmul (per-token and per-channel fp32 scales, bf16 out).
//
// Swap-AB: the weight tile is the MMA's M = 128 operand and the activation
// rows (M <= 16, zero-padded to 16 by the TMA box) are its N = 16 operand, so
// the tensor core consumes the packed weight image directly.  A work unit is
// one 128-row weight slab x two consecutive k-blocks (32 KB, contiguous in
// the packed image: one bulk copy).  The units are split evenly over all SMs
// (stream-K); a slab whose K range spans several CTAs is finished by the last
// CTA to arrive (atomic counter): it adds the others' int32 partials (exact,
// order-free) and runs the epilogue.  Nothing waits on another CTA.  Each
// counter word carries the call's tag (a per-process sequence number) next to
// its count, so whatever an earlier call -- or uninitialised memory -- left in
// the workspace is recognised as stale and restarted from 1: the workspace
// needs no clearing, and the kernel can start while the preceding kernel of
// the stream (the activation quantisation) is still running.
// Arithmetic identical to the large-M kernels and to the CPU oracle.
#include <cuda_bf16.h>

#include <atomic>

#include "gemm_common.cuh"

namespace w8a8 {
namespace {

constexpr int kUnitK = 2;                         // k-blocks per unit
constexpr int kUnitW = kUnitK * kTileBytes;       // 32 KB of weights per unit
constexpr int kQBox = kDecodeNT * kBK;            // 2 KB activation box per k-block
constexpr int kUnitQ = kUnitK * kQBox;            // 4 KB
constexpr int kDecodeStages = 5;                  // 5 x 36 KB in flight per SM

template <int STAGES>
struct DecodeSmem {
  static constexpr int kW = 0;
  static constexpr int kQ = STAGES * kUnitW;
  static constexpr int kBars = kQ + STAGES * kUnitQ;  // full, empty, tfull[2], tempty[2], done
  static constexpr int kMisc = kBars + (2 * STAGES + 5) * 8;
  static constexpr int kUsed = kMisc + 32;
  static constexpr int kAlloc = kUsed + 1024;
};

struct DecodeArgs {
  const uint8_t *packed_w;
  const float *a_scale;
  const float *w_scale;
  const uint16_t *bias;
  uint16_t *y;
  int M, N;
  int num_kb;          // k-blocks per 128-row slab
  int num_ku;          // units per slab = ceil(num_kb / kUnitK)
  int num_nb;          // 128-row slabs covering N
  int64_t units;       // num_nb * num_ku
  int max_contrib;     // partial slots per slab
  int32_t *partials;             // [num_nb][max_contrib][16][128]
  unsigned long long *counters;  // [num_nb]: (tag << 8) | arrivals
  unsigned long long tag;        // this call's tag (56 bits)
  int act;                       // w8a8_act applied after the dequantisation
  int *status;
};

__device__ __forceinline__ int64_t unit_begin(int64_t units, int grid, int c) {
  return units * c / grid;
}

// First CTA whose unit range contains unit u (ranges are [begin(c), begin(c+1))).
__device__ __forceinline__ int cta_of_unit(int64_t units, int grid, int64_t u) {
  int c = (int)((u * grid) / units);
  while (c + 1 < grid && unit_begin(units, grid, c + 1) <= u) ++c;
  while (c > 0 && unit_begin(units, grid, c) > u) --c;
  return c;
}

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_q, const DecodeArgs args) {
  using L = DecodeSmem<STAGES>;
  constexpr uint32_t kTmemCols = 32;  // two 16-column accumulators
  constexpr uint32_t kIdesc = idesc_i8(kBM, kDecodeNT);

  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sW = smem + L::kW;
  uint8_t *sQ = smem + L::kQ;
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kBars);
  uint64_t *empty = full + STAGES;
  uint64_t *tfull = empty + STAGES;
  uint64_t *tempty = tfull + 2;
  uint64_t *mma_done = tempty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
  volatile int *last_flag = reinterpret_cast<volatile int *>(smem + L::kMisc + 8);
  volatile int *seg_ok = reinterpret_cast<volatile int *>(smem + L::kMisc + 16);  // [2]
  volatile int *early_in = reinterpret_cast<volatile int *>(smem + L::kMisc + 24);  // [2]

  // Release the next kernel of the stream at once: the activation
  // quantisation of the next layer becomes resident beside this kernel and
  // waits on the device for it to finish, and the next layer's GEMM takes
  // each SM as soon as this kernel's CTA there exits, streaming its weights
  // while the last CTAs here still sum their partials.  (The large-M kernels
  // do not: the next quantisation's CTAs would crowd onto the SMs they leave
  // idle.)
  griddep_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
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

  const int64_t u_begin = unit_begin(args.units, gridDim.x, blockIdx.x);
  const int64_t u_end = unit_begin(args.units, gridDim.x, blockIdx.x + 1);
  const int nkb = args.num_kb, nku = args.num_ku;

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      const uint64_t evict_first = policy_evict_first();
      // A cursor walks this CTA's units: slab nb, first k-block kb0 and the
      // unit's weight pointer, which advances by kUnitK tiles (to the next
      // slab at a slab boundary).  As in the large-M kernels, no division
      // sits between a slot's release and its refill (0.5-1 % faster).
      struct Cur {
        int nb, kb0;
        const uint8_t *w;
      };
      auto at = [&](int64_t u) {
        Cur c;
        c.nb = (int)(u / nku);
        c.kb0 = (int)(u - (int64_t)c.nb * nku) * kUnitK;
        c.w = args.packed_w + ((size_t)c.nb * nkb + c.kb0) * kTileBytes;
        return c;
      };
      auto next = [&](Cur &c) {
        c.kb0 += kUnitK;
        if (c.kb0 >= nku * kUnitK) {
          c.kb0 = 0;
          ++c.nb;
          c.w = args.packed_w + (size_t)c.nb * nkb * kTileBytes;
        } else {
          c.w += (size_t)kUnitK * kTileBytes;
        }
      };
      auto c_nk = [&](const Cur &c) { return min(kUnitK, nkb - c.kb0); };
      auto c_weights = [&](const Cur &c, uint32_t s, int nk) {
        bulk_load_hint(sW + s * kUnitW, c.w, (uint32_t)(nk * kTileBytes), &full[s], evict_first);
      };
      auto c_acts = [&](const Cur &c, uint32_t s, int nk) {
        for (int h = 0; h < nk; ++h)
          tma_load_2d(sQ + s * kUnitQ + h * kQBox, &tmap_q, (c.kb0 + h) * kBK, 0, &full[s]);
      };
      bool ok = true;
      const int64_t n_units = u_end - u_begin;
      const uint32_t pre = n_units < STAGES ? (uint32_t)n_units : (uint32_t)STAGES;
      uint32_t issued = 0;
      if (n_units > 0) {
        Cur cur = at(u_begin);
        const Cur first = cur;
        // the weight stream does not depend on the preceding kernel
        for (uint32_t i = 0; i < pre; ++i) {
          const int nk = c_nk(cur);
          mbar_arrive_expect_tx(&full[i], (uint32_t)(nk * (kTileBytes + kQBox)));
          c_weights(cur, i, nk);
          next(cur);
        }
        griddep_wait();
        {
          Cur c = first;
          for (uint32_t i = 0; i < pre; ++i) {
            c_acts(c, i, c_nk(c));
            next(c);
          }
        }
        uint32_t s = 0, ph = 1;
        for (issued = pre; (int64_t)issued < n_units; ++issued) {
          const int nk = c_nk(cur);
          const uint32_t bytes = (uint32_t)(nk * (kTileBytes + kQBox));
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, args.status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], bytes);
          c_weights(cur, s, nk);
          c_acts(cur, s, nk);
          next(cur);
          if (++s == (uint32_t)STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      } else {
        griddep_wait();
      }
      if (!ok) {
        for (uint32_t sl = 0; sl < (uint32_t)STAGES && sl < issued; ++sl) {
          const uint32_t last = sl + ((issued - 1 - sl) / STAGES) * STAGES;
          volatile int no_abort = 0;
          (void)mbar_wait_bounded(&full[sl], (last / STAGES) & 1, &no_abort, args.status);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      uint32_t it = 0, seg = 0;
      bool ok = true;
      int64_t u = u_begin;
      while (ok && u < u_end) {
        const int nb = (int)(u / nku);
        const int64_t seg_end = min(u_end, (int64_t)(nb + 1) * nku);
        const uint32_t b = seg & 1, bph = (seg >> 1) & 1;
        if (!mbar_wait(&tempty[b], bph ^ 1, abort_flag, args.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * kDecodeNT;
        bool first = true;
        for (; u < seg_end; ++u, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, args.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int nk = min(kUnitK, nkb - (int)(u % nku) * kUnitK);
          for (int h = 0; h < nk; ++h) {
            const uint64_t a_desc = sw128_kmajor_desc(sW + s * kUnitW + h * kTileBytes);
            const uint64_t b_desc = sw128_kmajor_desc(sQ + s * kUnitQ + h * kQBox);
#pragma unroll
            for (int k = 0; k < kBK / 32; ++k)
              mma_i8(d_tmem, a_desc + 2 * k, b_desc + 2 * k, kIdesc,
                     (first && h == 0 && k == 0) ? 0u : 1u);
          }
          first = false;
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&tfull[b]);
        ++seg;
      }
      if (!ok) {
        mma_commit(mma_done);
        volatile int no_abort = 0;
        (void)mbar_wait_bounded(mma_done, 0, &no_abort, args.status);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..5): one output channel per thread ----
    // The four warps take every decision together: thread 0 of the group
    // waits on the barrier and publishes the outcome behind a named barrier,
    // so no warp can be left alone at a later named barrier.
    griddep_wait();  // a_scale may come from the preceding kernel
    const int quarter = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127
    float as[kDecodeNT];
#pragma unroll
    for (int m = 0; m < kDecodeNT; ++m) as[m] = m < args.M ? __ldg(args.a_scale + m) : 0.0f;
    uint32_t seg = 0;
    int64_t u = u_begin;
    while (u < u_end) {
      const int nb = (int)(u / nku);
      const int64_t slab_begin = (int64_t)nb * nku, slab_end = slab_begin + nku;
      const int64_t seg_end = min(u_end, slab_end);
      const bool whole = (u == slab_begin) && (seg_end == slab_end);
      const uint32_t b = seg & 1, bph = (seg >> 1) & 1;
      const int n_local = quarter * 32 + lane;  // TMEM lane = weight row in the slab
      const int n = nb * 128 + n_local;
      const float ws = n < args.N ? __ldg(args.w_scale + n) : 0.0f;
      const float bv =
          (args.bias && n < args.N) ? __uint_as_float((uint32_t)__ldg(args.bias + n) << 16) : 0.0f;
      // A slab split between CTAs: this CTA's rank among those covering it.
      // A CTA's last segment is usually the start of a slab whose other
      // parts its neighbours finished long before, at the start of their
      // ranges.  If every other contributor has already arrived, this CTA is
      // the last one: it takes their partials now, while its own MMAs run,
      // and adds them to its accumulators without publishing its own (no
      // stores, fence, tagged arrival or partial reads at the tail of the
      // kernel, which the next launch waits for).
      int contributors = 1, rank = 0;
      bool early = false;
      int32_t pre[kDecodeNT];
#pragma unroll
      for (int m = 0; m < kDecodeNT; ++m) pre[m] = 0;
      if (!whole) {
        const int first_cta = cta_of_unit(args.units, gridDim.x, slab_begin);
        const int last_cta = cta_of_unit(args.units, gridDim.x, slab_end - 1);
        contributors = last_cta - first_cta + 1;
        rank = blockIdx.x - first_cta;
        if (et == 0) {
          const unsigned long long v = ld_acquire_gpu(args.counters + nb);
          const bool in =
              (v >> 8) == args.tag && (uint32_t)(v & 0xFF) == (uint32_t)(contributors - 1);
          // no other arrival can follow: this call is done with the word
          if (in) args.counters[nb] = 0ull;
          // (its own word per buffer: threads may still read last_flag of
          // the previous segment)
          early_in[b] = in ? 1 : 0;
        }
        __syncwarp();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        early = early_in[b] != 0;
        if (early)
          for (int c = 0; c < contributors; ++c) {
            if (c == rank) continue;
            const int32_t *o = args.partials +
                               ((size_t)nb * args.max_contrib + c) * (128 * kDecodeNT) + n_local;
#pragma unroll
            for (int m = 0; m < kDecodeNT; ++m) pre[m] += __ldcg(o + m * 128);
          }
      }
      if (et == 0) seg_ok[b] = mbar_wait(&tfull[b], bph, abort_flag, args.status) ? 1 : 0;
      __syncwarp();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!seg_ok[b]) break;
      tc_fence_after();
      uint32_t r[kDecodeNT];
      tmem_ld_32x32b_x16(tmem_base + ((uint32_t)(quarter * 32) << 16) + b * kDecodeNT, r);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[b]);

      bool finish = whole;
      if (!whole && early) {
#pragma unroll
        for (int m = 0; m < kDecodeNT; ++m) r[m] = (uint32_t)((int32_t)r[m] + pre[m]);
        finish = true;
      } else if (!whole) {
        // The same check once more, now that this CTA's MMAs are done.
        if (et == 0) {
          const unsigned long long v = ld_acquire_gpu(args.counters + nb);
          const bool others_in =
              (v >> 8) == args.tag && (uint32_t)(v & 0xFF) == (uint32_t)(contributors - 1);
          // no other arrival can follow: this call is done with the word
          if (others_in) args.counters[nb] = 0ull;
          *last_flag = others_in ? 2 : 0;
        }
        __syncwarp();
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool others_in = *last_flag == 2;
        if (!others_in) {
          int32_t *slot = args.partials +
                          ((size_t)nb * args.max_contrib + rank) * (128 * kDecodeNT) + n_local;
#pragma unroll
          for (int m = 0; m < kDecodeNT; ++m) slot[m * 128] = (int32_t)r[m];
          __threadfence();
          __syncwarp();
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (et == 0) {
            const bool last =
                arrive_tagged(args.counters + nb, args.tag) == (uint32_t)contributors;
            // The last arrival of this call: nothing else touches the word in
            // this launch, so clear it.  A replayed CUDA graph relaunches with
            // the same tag and must find the count at zero, not at its total.
            if (last) args.counters[nb] = 0ull;
            *last_flag = last ? 1 : 0;
          }
          __syncwarp();
          asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        finish = *last_flag != 0;
        if (finish) {
          if (!others_in) __threadfence();
          int32_t sum[kDecodeNT];
#pragma unroll
          for (int m = 0; m < kDecodeNT; ++m) sum[m] = others_in ? (int32_t)r[m] : 0;
          for (int c = 0; c < contributors; ++c) {
            if (others_in && c == rank) continue;  // its own part is in r
            const int32_t *o = args.partials +
                               ((size_t)nb * args.max_contrib + c) * (128 * kDecodeNT) + n_local;
#pragma unroll
            for (int m = 0; m < kDecodeNT; ++m) sum[m] += __ldcg(o + m * 128);
          }
#pragma unroll
          for (int m = 0; m < kDecodeNT; ++m) r[m] = (uint32_t)sum[m];
        }
      }
      if (finish && n < args.N) {
#pragma unroll
        for (int m = 0; m < kDecodeNT; ++m) {
          if (m < args.M) {
            float t = dequant((int32_t)r[m], as[m], ws);
            if (args.bias) t = __fadd_rn(t, bv);
            t = apply_act(t, args.act);
            const __nv_bfloat16 h = __float2bfloat16_rn(t);
            args.y[(int64_t)m * args.N + n] = *reinterpret_cast<const uint16_t *>(&h);
          }
        }
      }
      u = seg_end;
      ++seg;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

FuncAttrOnce g_decode_smem_attr;

int64_t units_of(int64_t N, int64_t K) {
  const int64_t nkb = packed_cols(K) / 128;
  return (packed_rows(N) / 128) * ((nkb + kUnitK - 1) / kUnitK);
}

void geometry(int64_t N, int64_t K, int *grid, int *max_contrib) {
  const int64_t units = units_of(N, K);
  const int64_t g = std::min<int64_t>(units, sm_count());
  const int64_t per = units / g;  // shortest range of units a CTA gets
  const int64_t nku = (packed_cols(K) / 128 + kUnitK - 1) / kUnitK;
  *grid = (int)g;
  *max_contrib = (int)((nku + per - 1) / per + 1);
}

}  // namespace

int64_t decode_workspace_bytes(int64_t N, int64_t K) {
  int grid, mc;
  geometry(N, K, &grid, &mc);
  const int64_t nb = packed_rows(N) / 128;
  return round_up(nb * 8, 256) + nb * mc * 128 * kDecodeNT * 4;
}

bool use_decode_path(int64_t M) {
  const int p = forced_path();
  if (p == 2) return M <= kDecodeNT;
  if (p == 1 || p >= 3) return false;
  return M <= kDecodeNT;
}

w8a8_status launch_decode(const int8_t *q, const float *a_scale, const void *packed_w,
                          const float *w_scale, const void *bias, void *y, int64_t M,
                          int64_t N, int64_t K, void *workspace, cudaStream_t stream, bool pdl,
                          int act) {
  CUtensorMap tmap;
  if (!make_tmap_u8_2d(&tmap, q, (uint64_t)M, (uint64_t)K, (uint64_t)K, kDecodeNT, kBK))
    return W8A8_ERR_CUDA;
  int grid, mc;
  geometry(N, K, &grid, &mc);
  const int64_t nb = packed_rows(N) / 128;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  DecodeArgs a;
  a.packed_w = static_cast<const uint8_t *>(packed_w);
  a.a_scale = a_scale;
  a.w_scale = w_scale;
  a.bias = static_cast<const uint16_t *>(bias);
  a.y = static_cast<uint16_t *>(y);
  a.M = (int)M;
  a.N = (int)N;
  a.num_kb = (int)(packed_cols(K) / 128);
  a.num_ku = (a.num_kb + kUnitK - 1) / kUnitK;
  a.num_nb = (int)nb;
  a.units = nb * a.num_ku;
  a.max_contrib = mc;
  a.counters = reinterpret_cast<unsigned long long *>(ws);
  a.partials = reinterpret_cast<int32_t *>(ws + round_up(nb * 8, 256));
  a.tag = next_call_tag();
  a.act = act;
  a.status = status_word();
  if (!a.status) return W8A8_ERR_CUDA;
  cudaError_t e = cudaSuccess;
  using L = DecodeSmem<kDecodeStages>;
  auto k = decode_kernel<kDecodeStages>;
  if (g_decode_smem_attr.ensure([&] {
        return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
      }) != cudaSuccess)
    return W8A8_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = (size_t)L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, k, tmap, a);
  count_launch();
  return from_cuda(e);
}

}  // namespace w8a8
