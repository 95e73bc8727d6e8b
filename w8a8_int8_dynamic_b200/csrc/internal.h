// internal.h -- host-side helpers shared by the translation units of libw8a8.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "w8a8.h"

namespace w8a8 {

// Device pointer to this device's status word (0 = OK, else a w8a8_status).
int *status_word();

// Unique ID of the current CUDA context (false if none is current).
bool current_context_id(unsigned long long *id);

// One cached device address of a __device__ variable, valid for the context
// it was looked up in.
struct SymbolCache {
  std::mutex mu;
  bool valid = false;
  unsigned long long ctx_id = 0;
  void *addr = nullptr;
};

// The device address of `symbol` (the host-side name of a __device__
// variable) in the current context, from the cache while that context is the
// one it was looked up in, else from cudaGetSymbolAddress.
bool symbol_address(SymbolCache *cache, const void *symbol, void **out);

// A per-function setting (cudaFuncSetAttribute) made once per device and
// CUDA context: `set` runs unless it already succeeded in the context
// current now (by its process-wide unique ID, which a context created after
// a device reset or pushed by the caller does not share).  Any host thread
// may call it; two threads that find it unset both run `set`, which is
// idempotent.
struct FuncAttrOnce {
  static constexpr int kDevices = 64;
  std::atomic<unsigned long long> ctx_plus1[kDevices] = {};  // 0: not set
  template <typename F>
  cudaError_t ensure(F &&set) {
    int d = 0;
    unsigned long long id = 0;
    const bool have = cudaGetDevice(&d) == cudaSuccess && d >= 0 && d < kDevices &&
                      current_context_id(&id);
    if (have && ctx_plus1[d].load(std::memory_order_acquire) == id + 1) return cudaSuccess;
    const cudaError_t e = set();
    if (e == cudaSuccess && have) ctx_plus1[d].store(id + 1, std::memory_order_release);
    return e;
  }
};

// Number of SMs of the current device (cached per device).
int sm_count();

// Current device ordinal (cached per host thread).
int current_device();

// Counts one kernel launch (for the benchmark's launch accounting).
void count_launch(int n = 1);

// Path override set by w8a8_set_path: 0 auto, 1 large-M GEMM, 2 small-M.
int forced_path();

// A fresh 56-bit tag per call of a kernel that synchronises CTAs through
// workspace words (so words left by earlier calls never need clearing).
unsigned long long next_call_tag();

// 2-D tiled tensor map over a row-major uint8 matrix [rows, cols] with row
// stride ld bytes, box {box_cols, box_rows}, 128-byte swizzle, zero fill out
// of bounds.  Returns false if the driver rejects it.
bool make_tmap_u8_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                     uint64_t ld, uint32_t box_rows, uint32_t box_cols);

// Same, without swizzle: for the packed weight image, whose bytes are already
// in the tensor core's shared-memory order.
bool make_tmap_u8_2d_plain(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_rows, uint32_t box_cols);

// bf16 output y[M, N] for TMA stores: box 32 x 32, 64-byte swizzle.
bool make_tmap_out_bf16(CUtensorMap *map, const void *y, uint64_t M, uint64_t N);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline w8a8_status from_cuda(cudaError_t e) { return e == cudaSuccess ? W8A8_OK : W8A8_ERR_CUDA; }

// Size limits shared by the entry points.
constexpr int64_t kMaxK = 131072;

inline int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// Packed weight geometry: N padded to 256, K to 128; tiles of 128x128 bytes.
inline int64_t packed_rows(int64_t N) { return round_up(N, 256); }
inline int64_t packed_cols(int64_t K) { return round_up(K, 128); }

// GEMM launchers (gemm.cu).
// The next layer's quantisation fused with a GEMM (see GemmArgs::row_amax):
// per-row maxima (zeroed by the quantisation kernel ahead of the GEMM), per
// 128-row block call-tagged completion words, the call's tag, the codes and
// scales to form, and the exit count.
struct RowSignal {
  uint32_t *row_amax;
  unsigned long long *row_done;
  unsigned long long tag;
  int8_t *q_next;
  float *a_scale_next;
  unsigned long long *exit_word;
};
// pdl: a programmatic dependent of the preceding kernel; prefetch: (1-SM
// kernel) warm L2 with weights while waiting behind the quantisation kernel.
w8a8_status launch_scaled_mm(const int8_t *q, const float *a_scale, const void *packed_w,
                             const float *w_scale, const void *bias, void *out, bool out_i32,
                             int64_t M, int64_t N, int64_t K, cudaStream_t stream, bool pdl,
                             int act = W8A8_ACT_NONE, bool prefetch = false,
                             const RowSignal *sig = nullptr);
// Workspace of w8a8_linear: codes, scales and (small M) the decode partials.
int64_t linear_workspace_bytes(int64_t M, int64_t N, int64_t K);
// 2-SM (CTA pair) GEMM with the bf16 epilogue (gemm2sm.cu); bn = 256 or 128.
w8a8_status launch_gemm2sm(const int8_t *q, const float *a_scale, const void *packed_w,
                           const float *w_scale, const void *bias, void *y, int64_t M, int64_t N,
                           int64_t K, cudaStream_t stream, bool pdl, int bn,
                           int act = W8A8_ACT_NONE, const RowSignal *sig = nullptr);
int64_t pair_tiles(int64_t M, int64_t N, int bn);
int64_t pair_full_tiles(int64_t tiles, int64_t pairs);
// Small-M weight-streaming kernel (decode.cu).
int64_t decode_workspace_bytes(int64_t N, int64_t K);
bool use_decode_path(int64_t M);
w8a8_status launch_decode(const int8_t *q, const float *a_scale, const void *packed_w,
                          const float *w_scale, const void *bias, void *y, int64_t M,
                          int64_t N, int64_t K, void *workspace, cudaStream_t stream, bool pdl,
                          int act = W8A8_ACT_NONE);
// Quantisation launcher (quant.cu).  ahead_of_gemm: the launch is followed by
// a GEMM launched as its programmatic dependent (the layer).  zero_rows
// (nullable): a per-row word the kernel sets to 0 (the row maxima of a GEMM
// with the next layer's quantisation fused in).
w8a8_status launch_quant(const void *x, int64_t M, int64_t K, int64_t ldx, int8_t *q,
                         float *a_scale, cudaStream_t stream, bool ahead_of_gemm,
                         uint32_t *zero_rows = nullptr);


}  // namespace w8a8
