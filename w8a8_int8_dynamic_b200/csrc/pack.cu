// pack.cu -- load-time weight repack: int8 W[N, K] -> tensor-core tile image.
//
// Source: "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
// Round two, kernel-path verification: the layer's weights are transposed
// and repacked once as they are loaded, then applied, and the loaded weights
// (the fused Q/K/V ones too) are checked bit for bit.  The layout is this
// library's own.
//
// Layout: N padded to Np = round_up(N, 256), K to Kp = round_up(K, 128).
// Tiles of 128 rows (n) x 128 bytes (k), tile (nb, kb) at byte offset
// (nb * Kp/128 + kb) * 16384, so the k-blocks of one 128-row slab are
// contiguous.  Inside a tile, row r occupies bytes [128 r, 128 r + 128) and
// its 16-byte chunk j is stored at chunk position j XOR (r mod 8): exactly
// the K-major, 128-byte-swizzled shared-memory image that tcgen05.mma reads
// through a SWIZZLE_128B descriptor (8-row atoms, 1024-byte stride), so the
// GEMM moves whole tiles with one 16 KB bulk copy and no tensor map.
// Padding bytes are zero, so padded K columns and N rows add nothing.
#include "internal.h"

namespace w8a8 {
namespace {

// One thread per 16-byte chunk of the packed buffer (coalesced writes; the
// 8 threads of one row read one contiguous 128-byte row segment).
// `flip` is XORed into every source word: 0 for int8 input, 0x80808080 for
// the biased-uint8 int32 storage (byte (w + 128) XOR 0x80 is w as int8).
__global__ void pack_kernel(const int8_t *__restrict__ w, int64_t N, int64_t K, int64_t kblocks,
                            int64_t total_chunks, uint32_t flip, uint4 *__restrict__ out) {
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_chunks;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = o >> 10;          // 1024 chunks per tile
    const int r = (int)((o >> 3) & 127);   // row inside the tile
    const int pos = (int)(o & 7);          // stored chunk position
    const int j = pos ^ (r & 7);           // logical chunk
    const int64_t n = (tile / kblocks) * 128 + r;
    const int64_t k = (tile % kblocks) * 128 + j * 16;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (n < N && k < K) {
      v = *reinterpret_cast<const uint4 *>(w + n * K + k);
      v.x ^= flip;
      v.y ^= flip;
      v.z ^= flip;
      v.w ^= flip;
    }
    out[o] = v;
  }
}

__global__ void unpack_kernel(const uint4 *__restrict__ in, int64_t N, int64_t K,
                              int64_t kblocks, int64_t total_chunks, int8_t *__restrict__ w) {
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < total_chunks;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t tile = o >> 10;
    const int r = (int)((o >> 3) & 127);
    const int pos = (int)(o & 7);
    const int j = pos ^ (r & 7);
    const int64_t n = (tile / kblocks) * 128 + r;
    const int64_t k = (tile % kblocks) * 128 + j * 16;
    if (n < N && k < K) *reinterpret_cast<uint4 *>(w + n * K + k) = in[o];
  }
}

w8a8_status launch_pack(const int8_t *w, int64_t N, int64_t K, void *packed, uint32_t flip,
                        cudaStream_t stream) {
  const int64_t chunks = packed_rows(N) * packed_cols(K) / 16;
  const int64_t blocks = std::min<int64_t>((chunks + 255) / 256, (int64_t)sm_count() * 16);
  pack_kernel<<<(unsigned)blocks, 256, 0, stream>>>(w, N, K, packed_cols(K) / 128, chunks, flip,
                                                    static_cast<uint4 *>(packed));
  count_launch();
  return from_cuda(cudaGetLastError());
}

w8a8_status check_weight_shape(int64_t N, int64_t K) {
  if (N < 1 || K < 1) return W8A8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > kMaxK || N % 8 != 0 || N > (int64_t)1 << 30)
    return W8A8_ERR_UNSUPPORTED_SHAPE;
  return W8A8_OK;
}

}  // namespace
}  // namespace w8a8

using namespace w8a8;

extern "C" {

w8a8_status w8a8_packed_weight_bytes(int64_t N, int64_t K, size_t *bytes) {
  if (!bytes) return W8A8_ERR_INVALID_ARG;
  const w8a8_status st = check_weight_shape(N, K);
  if (st != W8A8_OK) return st;
  *bytes = (size_t)(packed_rows(N) * packed_cols(K));
  return W8A8_OK;
}

w8a8_status w8a8_pack_weight(const int8_t *w, int64_t N, int64_t K, void *packed,
                             size_t packed_bytes, w8a8_stream_t stream) {
  if (!w || !packed) return W8A8_ERR_INVALID_ARG;
  const w8a8_status st = check_weight_shape(N, K);
  if (st != W8A8_OK) return st;
  if (!aligned16(w) || !aligned16(packed)) return W8A8_ERR_ALIGNMENT;
  const int64_t need = packed_rows(N) * packed_cols(K);
  if ((int64_t)packed_bytes < need) return W8A8_ERR_BUFFER_TOO_SMALL;
  return launch_pack(w, N, K, packed, 0u, reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_pack_weight_int32(const int32_t *w_i32, int64_t N, int64_t K, void *packed,
                                   size_t packed_bytes, w8a8_stream_t stream) {
  if (!w_i32 || !packed) return W8A8_ERR_INVALID_ARG;
  const w8a8_status st = check_weight_shape(N, K);
  if (st != W8A8_OK) return st;
  if (!aligned16(w_i32) || !aligned16(packed)) return W8A8_ERR_ALIGNMENT;
  const int64_t need = packed_rows(N) * packed_cols(K);
  if ((int64_t)packed_bytes < need) return W8A8_ERR_BUFFER_TOO_SMALL;
  return launch_pack(reinterpret_cast<const int8_t *>(w_i32), N, K, packed, 0x80808080u,
                     reinterpret_cast<cudaStream_t>(stream));
}

w8a8_status w8a8_unpack_weight(const void *packed, int64_t N, int64_t K, int8_t *w,
                               w8a8_stream_t stream) {
  if (!w || !packed) return W8A8_ERR_INVALID_ARG;
  const w8a8_status st = check_weight_shape(N, K);
  if (st != W8A8_OK) return st;
  if (!aligned16(w) || !aligned16(packed)) return W8A8_ERR_ALIGNMENT;
  const int64_t chunks = packed_rows(N) * packed_cols(K) / 16;
  const int64_t blocks = std::min<int64_t>((chunks + 255) / 256, (int64_t)sm_count() * 16);
  unpack_kernel<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4 *>(packed), N, K, packed_cols(K) / 128, chunks, w);
  count_launch();
  return from_cuda(cudaGetLastError());
}

}  // extern "C"
