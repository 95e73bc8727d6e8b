// noalloc.cu -- the whole W8A8 layer (quantise + GEMM + epilogue) for callers
// that cannot hand the library a workspace.
//
// Some callers cannot allocate device memory at the moment they run a layer:
// a plugin whose host framework owns every byte of device memory through its
// own pool and forbids cudaMalloc from inside execution callbacks, or a
// latency-critical loop where the implicit device-wide synchronisation of
// cudaMalloc / cudaFree is not acceptable.  w8a8_linear needs a caller-provided
// workspace for the quantised activations, their scales and (for small M) the
// split-K partials; this entry point instead uses one scratch array that lives
// in this library's device memory for as long as the library is loaded.
//
// The array is a file-scope __device__ variable, so each GPU that loads the
// library holds kNoAllocScratchBytes of it until the process exits.  Host code
// cannot use the array's name as a device address (it is a host-side stand-in),
// so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and keeps it.  The kept
// address belongs to the CUDA context it was looked up in: it is reused only
// while that same context (by its process-wide unique ID) is current, and
// looked up again after a device reset or under another context.
#include <mutex>

#include "internal.h"

namespace w8a8 {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device

__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
struct ScratchSlot {
  bool valid;
  unsigned long long ctx_id;
  void *addr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;  // guards every read and write of g_scratch

// Device address of the scratch array in the current context (set-up on the
// first call in each context).
w8a8_status scratch_address(void **out) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return W8A8_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  ScratchSlot &slot = g_scratch[d];
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  if (have_id && slot.valid && slot.ctx_id == id) {
    *out = slot.addr;
    return W8A8_OK;
  }
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return W8A8_ERR_CUDA;
  if (!have_id) have_id = current_context_id(&id);  // the lookup may have created it
  slot.valid = have_id;
  slot.ctx_id = id;
  slot.addr = p;
  *out = p;
  return W8A8_OK;
}

}  // namespace
}  // namespace w8a8

using namespace w8a8;

extern "C" size_t w8a8_linear_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

extern "C" w8a8_status w8a8_linear_noalloc(const void *x, int64_t ldx, const void *packed_w,
                                           const float *w_scale, const void *bias, void *y,
                                           int64_t M, int64_t N, int64_t K,
                                           w8a8_stream_t stream) {
  size_t need = 0;
  const w8a8_status st = w8a8_linear_workspace_bytes(M, N, K, &need);
  if (st != W8A8_OK) return st;
  if (need > kNoAllocScratchBytes) return W8A8_ERR_BUFFER_TOO_SMALL;
  void *scratch = nullptr;
  const w8a8_status sa = scratch_address(&scratch);
  if (sa != W8A8_OK) return sa;
  // Everything the layer reads from the scratch is written first in the same
  // call (codes, scales, partials), and the small-M split-K counters carry a
  // per-call tag, so what a previous call left there does not matter.
  return w8a8_linear(x, ldx, packed_w, w_scale, bias, y, M, N, K, scratch, kNoAllocScratchBytes,
                     stream);
}
