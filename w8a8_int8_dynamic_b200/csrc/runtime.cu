// runtime.cu -- status word, error polling, device queries, tensor-map
// encoding and the bounded-wait self-test of libw8a8.
#include <atomic>
#include <cudaTypedefs.h>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace w8a8 {

// One status word per device (module globals are instantiated per device).
__device__ int g_status_word;

namespace {
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::mutex g_mu;
std::atomic<int64_t> g_launches{0};
std::atomic<int> g_forced_path{0};
std::atomic<unsigned long long> g_call_tag{0};
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Driver entry points that identify the current CUDA context.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
std::once_flag g_ctx_fns_once;
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

SymbolCache g_status_cache;
}  // namespace

int current_device() {
  int d = 0;
  cudaGetDevice(&d);
  return d;
}

bool current_context_id(unsigned long long *id) {
  std::call_once(g_ctx_fns_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(fn);
  });
  if (!g_ctx_get_current || !g_ctx_get_id) return false;
  CUcontext c = nullptr;
  if (g_ctx_get_current(&c) != CUDA_SUCCESS || !c) return false;
  return g_ctx_get_id(c, id) == CUDA_SUCCESS;
}

// The device address of a __device__ variable in the current context.  A
// cached address is reused only while the same context (by its process-wide
// unique ID, which a context created after a device reset does not share) is
// current; otherwise it is looked up again.  The mutex covers every read and
// write of the cache.
bool symbol_address(SymbolCache *cache, const void *symbol, void **out) {
  std::lock_guard<std::mutex> lk(cache->mu);
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  if (have_id && cache->valid && cache->ctx_id == id) {
    *out = cache->addr;
    return true;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess || !p) return false;
  // the lookup may itself have made the device's primary context current
  if (!have_id) have_id = current_context_id(&id);
  cache->valid = have_id;
  cache->ctx_id = id;
  cache->addr = p;
  *out = p;
  return true;
}

int *status_word() {
  void *p = nullptr;
  if (!symbol_address(&g_status_cache, reinterpret_cast<const void *>(&g_status_word), &p))
    return nullptr;
  return static_cast<int *>(p);
}

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  int n = g_sm_count[d].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    if (n <= 0) n = 148;
    g_sm_count[d].store(n, std::memory_order_relaxed);
  }
  return n;
}

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int forced_path() { return g_forced_path.load(std::memory_order_relaxed); }

unsigned long long next_call_tag() {
  return (g_call_tag.fetch_add(1, std::memory_order_relaxed) + 1) & ((1ull << 56) - 1);
}

static bool encode_u8_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                         uint64_t ld, uint32_t box_rows, uint32_t box_cols,
                         CUtensorMapSwizzle swizzle) {
  if (!g_encode) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void *fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return false;
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {ld};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                     uint64_t ld, uint32_t box_rows, uint32_t box_cols) {
  return encode_u8_2d(map, base, rows, cols, ld, box_rows, box_cols, CU_TENSOR_MAP_SWIZZLE_128B);
}

bool make_tmap_u8_2d_plain(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_rows, uint32_t box_cols) {
  return encode_u8_2d(map, base, rows, cols, ld, box_rows, box_cols, CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool make_tmap_out_bf16(CUtensorMap *map, const void *y, uint64_t M, uint64_t N) {
  if (!g_encode) {
    CUtensorMap tmp;
    if (!encode_u8_2d(&tmp, y, 1, 16, 16, 1, 16, CU_TENSOR_MAP_SWIZZLE_NONE)) return false;
  }
  const cuuint64_t dims[2] = {N, M};
  const cuuint64_t strides[1] = {N * 2};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(y),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Waits on a barrier that nothing arrives at; the bounded wait must give up.
__global__ void selftest_wait_kernel(int *status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: the single expected arrival never comes
    (void)mbar_wait_bounded(&bar, 0, &abort_flag, status, limit_ns);
  }
  __syncthreads();
}

// The int8 tensor-core rate with no memory traffic, the ceiling the GEMMs'
// fractions are read against beside the measured bf16 rate: every CTA (one
// per SM) issues `iters` groups of four tcgen05.mma.cta_group::1.kind::i8
// (M = 128, N = 256, K = 32) from fixed shared-memory tiles into one TMEM
// accumulator, then waits (bounded) for them.  The operand bytes are an
// arbitrary pattern of small values (not zeros, which toggle less); the
// int32 sums wrap and are never read.
constexpr int kRateN = 256;
constexpr int kRateSmem = 16384 + kRateN * 128 + 16 + 1024;

__global__ void __launch_bounds__(128, 1) selftest_mma_rate_kernel(int iters, int *status) {
  extern __shared__ uint8_t raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  uint8_t *sA = sm, *sB = sm + 16384;  // 128 x 128 and 256 x 128 int8 tiles (SW128 images)
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + 16384 + kRateN * 128);
  uint32_t *slot = reinterpret_cast<uint32_t *>(bar + 1);
  __shared__ int abort_flag;
  for (int i = threadIdx.x; i < (16384 + kRateN * 128) / 4; i += blockDim.x)
    reinterpret_cast<uint32_t *>(sm)[i] = 0x01010101u * (((uint32_t)i * 2654435761u) >> 29);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  fence_proxy_async_smem();  // the operand bytes, before the tensor core reads them
  if (threadIdx.x < 32) tmem_alloc(slot, kRateN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  if (threadIdx.x == 0) {
    const uint64_t ad = sw128_kmajor_desc(sA), bd = sw128_kmajor_desc(sB);
    constexpr uint32_t id = idesc_i8(128, kRateN);
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int k = 0; k < 4; ++k) mma_i8(tmem, ad + 2 * k, bd + 2 * k, id, (it | k) != 0);
    mma_commit(bar);
    (void)mbar_wait_bounded(bar, 0, &abort_flag, status);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, kRateN);
  }
}

FuncAttrOnce g_rate_smem_attr;

}  // namespace w8a8

using namespace w8a8;

extern "C" {

const char *w8a8_status_string(int status) {
  switch (status) {
    case W8A8_OK: return "W8A8_OK";
    case W8A8_ERR_INVALID_ARG: return "W8A8_ERR_INVALID_ARG";
    case W8A8_ERR_ALIGNMENT: return "W8A8_ERR_ALIGNMENT";
    case W8A8_ERR_UNSUPPORTED_SHAPE: return "W8A8_ERR_UNSUPPORTED_SHAPE";
    case W8A8_ERR_CUDA: return "W8A8_ERR_CUDA";
    case W8A8_ERR_TIMEOUT: return "W8A8_ERR_TIMEOUT";
    case W8A8_ERR_BUFFER_TOO_SMALL: return "W8A8_ERR_BUFFER_TOO_SMALL";
    default: return "W8A8_ERR_UNKNOWN";
  }
}

int w8a8_abi_version(void) { return (1 << 16) | 1; }

w8a8_status w8a8_set_path(int path) {
  if (path < 0 || path > 7 || path == 6) return W8A8_ERR_INVALID_ARG;
  g_forced_path.store(path);
  return W8A8_OK;
}

int64_t w8a8_launch_count(void) { return g_launches.load(); }

w8a8_status w8a8_poll_status(w8a8_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int *sw = status_word();
  if (!sw) return W8A8_ERR_CUDA;
  int host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, sw, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return W8A8_ERR_CUDA;
  if (host != 0) {
    const int zero = 0;
    e = cudaMemcpyAsync(sw, &zero, sizeof(int), cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return W8A8_ERR_CUDA;
    return static_cast<w8a8_status>(host);
  }
  return W8A8_OK;
}

w8a8_status w8a8_selftest_int8_mma_rate(int64_t iters, w8a8_stream_t stream, double *tops) {
  // At most 2e5 groups (about 55 ms of MMAs at 1.9 GHz), so the loop ends well
  // inside the kernel's one bounded wait (1 s) even at a much lower clock.
  if (!tops || iters < 1 || iters > 200000) return W8A8_ERR_INVALID_ARG;
  int *sw = status_word();
  if (!sw) return W8A8_ERR_CUDA;
  if (g_rate_smem_attr.ensure([] {
        return cudaFuncSetAttribute(selftest_mma_rate_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kRateSmem);
      }) != cudaSuccess)
    return W8A8_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = sm_count();
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
    if (e0) cudaEventDestroy(e0);
    return W8A8_ERR_CUDA;
  }
  selftest_mma_rate_kernel<<<sms, 128, kRateSmem, s>>>(64, sw);  // warm-up
  cudaEventRecord(e0, s);
  selftest_mma_rate_kernel<<<sms, 128, kRateSmem, s>>>((int)iters, sw);
  cudaEventRecord(e1, s);
  count_launch(2);
  cudaError_t e = cudaEventSynchronize(e1);
  float ms = 0.0f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (e != cudaSuccess) return W8A8_ERR_CUDA;
  *tops = ms > 0.0f ? (double)sms * (double)iters * 4.0 * 2.0 * 128.0 * kRateN * 32.0 /
                          (ms * 1e-3) / 1e12
                    : 0.0;
  return from_cuda(cudaGetLastError());
}

w8a8_status w8a8_selftest_wait_timeout(int64_t timeout_ns, w8a8_stream_t stream) {
  if (timeout_ns < 1000) timeout_ns = 1000;
  if (timeout_ns > 5000000000LL) timeout_ns = 5000000000LL;
  int *sw = status_word();
  if (!sw) return W8A8_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      sw, static_cast<uint64_t>(timeout_ns));
  count_launch();
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
