/*
 * w8a8.h -- C ABI of libw8a8.so: W8A8 int8-dynamic linear layers for NVIDIA
 * B200 (sm_100a).
 *
 * The method (sources by page title and section):
 *   "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090",
 *   Round two: int8 weights with fp32 per-output-channel scales, int8
 *   activations with one symmetric scale per token computed at run time, an
 *   int8 scaled matmul, and weights transposed and repacked once at load
 *   time, then applied, in fused Q/K/V and row-parallel layers as well.  "INT8 Quant for Dual-Max Recipe": int8 x int8 on
 *   the integer tensor cores with no dequantisation of the weights.
 *   "Online Quantization", Parameters: activation_scheme "dynamic".
 *
 * Arithmetic (identical, bit for bit, to the CPU oracle of this repository):
 *   a_scale[m] = amax_k |x[m,k]| / 127                (fp32, IEEE division)
 *   q[m,k]     = clamp(rint_half_even(x[m,k] / a_scale[m]), -127, 127)
 *                (q = 0 and a_scale = 0 for a row whose amax is 0)
 *   acc[m,n]   = sum_k q[m,k] * w[n,k]                 (exact int32)
 *   y[m,n]     = bf16_rne(((float)acc * a_scale[m]) * w_scale[n] + bias[n])
 *                (each step one fp32 operation rounded to nearest even)
 *
 * Conventions for every entry point:
 *   - Pointers marked "device" are CUDA device pointers of the current
 *     device; the caller allocates and owns them.  The library allocates no
 *     device memory per call (it keeps one 4-byte status word per device).
 *   - Matrices are row-major.  x: bf16 [M, K] with row stride ldx elements;
 *     q: int8 [M, K] dense; w: int8 [N, K] (K contiguous, i.e. out x in);
 *     y: bf16 [M, N] dense.  bf16 is passed as raw 16-bit storage.
 *   - All work is enqueued on `stream` (NULL = legacy default stream) and is
 *     asynchronous; no entry point synchronises except w8a8_poll_status.
 *   - Argument checks run on the host before any launch; on failure nothing
 *     is launched and the status says why.  A launch failure returns
 *     W8A8_ERR_CUDA.  Kernels never trap: a device-side wait that exceeds
 *     its time limit (about one second) records W8A8_ERR_TIMEOUT in the
 *     device status word, which w8a8_poll_status reports.
 *   - Shape limits: 1 <= M <= 2^31-1, 1 <= N, 16 <= K <= 131072, K % 16 == 0
 *     (16-byte rows for TMA), N % 8 == 0 (16-byte output rows), all pointers
 *     16-byte aligned.  K <= 131072 keeps |acc| <= 131072*127*128 < 2^31.
 *   - Calls that share buffers and overlap on the GPU race; use one stream
 *     or events.
 */
#ifndef W8A8_H_
#define W8A8_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *w8a8_stream_t;

typedef enum w8a8_status {
  W8A8_OK = 0,
  W8A8_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum */
  W8A8_ERR_ALIGNMENT = 2,         /* pointer or stride not 16-byte aligned */
  W8A8_ERR_UNSUPPORTED_SHAPE = 3, /* K % 16, N % 8, K range, M range */
  W8A8_ERR_CUDA = 4,              /* a CUDA runtime / launch error */
  W8A8_ERR_TIMEOUT = 5,           /* a device-side wait gave up (kernel output invalid) */
  W8A8_ERR_BUFFER_TOO_SMALL = 6   /* packed or workspace buffer too small */
} w8a8_status;

/* Activation applied to the layer output inside the GEMM epilogue.
 * W8A8_ACT_GELU_TANH: the output is bf16(GELU_tanh(bf16(y))), i.e. exactly
 * the result of the plain layer followed by w8a8_gelu_tanh, without the
 * round trip of y through memory.  GELU_tanh(v) = 0.5 v (1 + tanh(sqrt(2/pi)
 * (v + 0.044715 v^3))) in fp32; it joins the up- and down-projections of a
 * transformer MLP and is not part of the quantisation method. */
typedef enum {
  W8A8_ACT_NONE = 0,
  W8A8_ACT_GELU_TANH = 1
} w8a8_act;

/* Human-readable name of a status code (static string, never NULL). */
const char *w8a8_status_string(int status);

/* ABI version of this header: (major << 16) | minor. */
int w8a8_abi_version(void);

/* ---- step 1: dynamic per-token activation quantisation ------------------
 * Source: "Issue 5 probe ...", Round two (int8 activations, one symmetric
 * scale per token computed at run time; op scaled_int8_quant); "Online
 * Quantization", Parameters.
 *   x       device, bf16 [M, K], row stride ldx >= K elements (ldx % 8 == 0)
 *   q       device, int8 [M, K] dense (output)
 *   a_scale device, fp32 [M]   (output)
 * One pass over x: 2*M*K bytes read, M*K + 4*M bytes written. */
w8a8_status w8a8_quant_act(const void *x, int64_t M, int64_t K, int64_t ldx,
                           int8_t *q, float *a_scale, w8a8_stream_t stream);

/* Static (calibrated) activation scale, the other activation scheme of
 * "Online Quantization", Parameters: one fp32 scale for the whole tensor,
 * computed offline.  code = clamp(rint_half_even(x / scale), -127, 127)
 * (values outside the calibrated range saturate); a scale that is not > 0
 * (zero, negative, NaN) gives all codes 0 and a_scale 0.
 *   x       device, bf16 [M, K], row stride ldx >= K elements (ldx % 8 == 0)
 *   scale   device, one fp32 (4-byte aligned); read by the kernel, so a new
 *           calibration needs no host synchronisation
 *   q       device, int8 [M, K] dense (output)
 *   a_scale device, fp32 [M] (output; may be NULL): every entry = the scale
 *           used, so w8a8_scaled_mm applies it unchanged
 * Same shape rules and errors as w8a8_quant_act. */
w8a8_status w8a8_quant_act_static(const void *x, int64_t M, int64_t K, int64_t ldx,
                                  const float *scale, int8_t *q, float *a_scale,
                                  w8a8_stream_t stream);

/* ---- step 2 (load time): weight repack ------------------------------------
 * Source: "Issue 5 probe ...", Round two, kernel-path verification (weights
 * transposed and repacked once at load time); the layout is this library's own:
 * 128x128-byte tiles, each the K-major 128-byte-swizzled shared-memory image
 * the tensor core reads, N padded to 256 and K to 128 with zeros.
 *   Byte size of the packed buffer for an [N, K] weight: */
w8a8_status w8a8_packed_weight_bytes(int64_t N, int64_t K, size_t *bytes);

/*   w      device, int8 [N, K] row-major (K contiguous)
 *   packed device, packed_bytes >= w8a8_packed_weight_bytes(N, K)
 * Every byte of `packed` is written (padding with zeros).  Fused Q/K/V:
 * concatenate the three [hidden, K] blocks along N (and their scales) and
 * pack once; the output's column slices are the three projections. */
w8a8_status w8a8_pack_weight(const int8_t *w, int64_t N, int64_t K,
                             void *packed, size_t packed_bytes,
                             w8a8_stream_t stream);

/* Inverse of w8a8_pack_weight (test and inspection use): packed -> w [N, K]. */
w8a8_status w8a8_unpack_weight(const void *packed, int64_t N, int64_t K,
                               int8_t *w, w8a8_stream_t stream);

/* ---- load time: online weight quantisation + repack in one pass -------------
 * Source: "Online Quantization", Overview (quantised weights and their scales
 * computed while the model loads, from a higher-precision checkpoint);
 * "Issue 5 probe ...", Round one (per-output-channel symmetric int8 weights).
 * Per output channel n: w_scale[n] = max_k |W[n,k]| / 127 (IEEE fp32
 * division), code = rint_half_even(W[n,k] / w_scale[n]) in [-127, 127]; an
 * all-zero channel gets scale 0 and codes 0.  Same rule as w8a8_quant_act
 * applied to the rows of W.
 *   w       device, bf16 [N, K] row-major
 *   packed  device, packed_bytes >= w8a8_packed_weight_bytes(N, K); every byte
 *           written, same image as w8a8_pack_weight of the int8 codes
 *   w_scale device, fp32 [N] (output)
 * Shape rules as w8a8_pack_weight; w, packed, w_scale 16-byte aligned. */
w8a8_status w8a8_quant_pack_weight(const void *w, int64_t N, int64_t K,
                                   void *packed, size_t packed_bytes,
                                   float *w_scale, w8a8_stream_t stream);

/* ---- load time: repack from compressed-tensors int32 storage ----------------
 * Source: "Issue 5 probe ...", Artifact (weights stored with pack_to_int32:
 * four unsigned bytes, each weight + 128, to an int32 word).  Bit order (not printed there; this
 * library's reading): element 4j+i of a row is bits [8i, 8i+8) of word j,
 * holding the unsigned byte (w + 128).
 *   w_i32   device, int32 [N, K/4] row-major, 16-byte aligned
 *   packed  as w8a8_pack_weight; the result equals w8a8_pack_weight of the
 *           decoded int8 [N, K] weight. */
w8a8_status w8a8_pack_weight_int32(const int32_t *w_i32, int64_t N, int64_t K,
                                   void *packed, size_t packed_bytes,
                                   w8a8_stream_t stream);

/* ---- steps 3+4: int8 GEMM with the dequantising epilogue -----------------
 * Source: "Issue 5 probe ...", Round two (op cutlass_scaled_mm: int8 x int8
 * with per-token and per-channel fp32 scales); "INT8 Quant for Dual-Max
 * Recipe" (native int8 tensor-core path, no weight dequantisation).
 *   q        device, int8 [M, K] dense (from w8a8_quant_act)
 *   a_scale  device, fp32 [M]
 *   packed_w device, from w8a8_pack_weight(N, K)
 *   w_scale  device, fp32 [N]
 *   bias     device, bf16 [N], or NULL for no bias
 *   y        device, bf16 [M, N] (output)
 *   workspace device scratch of ws_bytes >= w8a8_scaled_mm_workspace_bytes,
 *            or NULL (16-byte aligned; contents on entry do not matter).  For
 *            M <= 16 it holds the weight-streaming kernel's int32 split-K
 *            partials and call-tagged counters; the size query returns 0
 *            for larger M, whose kernels need none.  With NULL (or too
 *            small), M <= 16 falls back to the large-M kernels.
 * All kernels give bit-identical results (the partials are summed exactly
 * in int32 before the scale arithmetic). */
w8a8_status w8a8_scaled_mm_workspace_bytes(int64_t M, int64_t N, int64_t K,
                                           size_t *bytes);
w8a8_status w8a8_scaled_mm(const int8_t *q, const float *a_scale,
                           const void *packed_w, const float *w_scale,
                           const void *bias, void *y, int64_t M, int64_t N,
                           int64_t K, void *workspace, size_t ws_bytes,
                           w8a8_stream_t stream);

/* w8a8_scaled_mm with an activation (w8a8_act) applied in the epilogue:
 * act = W8A8_ACT_GELU_TANH writes bf16(GELU_tanh(y)) instead of y (the
 * fused form of the MLP up-projection followed by its GELU).  Any other
 * value than the w8a8_act members -> W8A8_ERR_INVALID_ARG. */
w8a8_status w8a8_scaled_mm_act(const int8_t *q, const float *a_scale,
                               const void *packed_w, const float *w_scale,
                               const void *bias, void *y, int64_t M, int64_t N,
                               int64_t K, int act, void *workspace,
                               size_t ws_bytes, w8a8_stream_t stream);

/* The int32 accumulators acc[M, N] of the same GEMM, without the epilogue
 * (test and inspection use; acc device, int32 [M, N]). */
w8a8_status w8a8_scaled_mm_i32(const int8_t *q, const void *packed_w,
                               int32_t *acc, int64_t M, int64_t N, int64_t K,
                               w8a8_stream_t stream);

/* ---- the whole layer: quantise + GEMM + epilogue --------------------------
 * Source: "Issue 5 probe ...", Round two (the layer path: the activation
 * quantisation feeds the scaled matmul).  Two launches on `stream`; the GEMM
 * is launched as a programmatic dependent of the quantisation so that its
 * set-up overlaps the quantisation's tail.
 *   x         device, bf16 [M, K], row stride ldx
 *   workspace device, ws_bytes >= w8a8_linear_workspace_bytes(M, N, K); holds
 *             q and a_scale (each rounded up to 256 bytes), then for M <= 16
 *             the small-M kernel's partials (see w8a8_scaled_mm).  Its
 *             contents on entry do not matter.
 * N-D activations [..., K] are flattened by the caller to [M, K] and y is
 * viewed back as [..., N] (the "Diffusion Quantization Reference", GGUF
 * rules and the output-rank failure in "Common Failures"). */
w8a8_status w8a8_linear_workspace_bytes(int64_t M, int64_t N, int64_t K,
                                        size_t *bytes);
w8a8_status w8a8_linear(const void *x, int64_t ldx, const void *packed_w,
                        const float *w_scale, const void *bias, void *y,
                        int64_t M, int64_t N, int64_t K, void *workspace,
                        size_t ws_bytes, w8a8_stream_t stream);

/* w8a8_linear with an activation applied in the epilogue (see
 * w8a8_scaled_mm_act); same workspace. */
w8a8_status w8a8_linear_act(const void *x, int64_t ldx, const void *packed_w,
                            const float *w_scale, const void *bias, void *y,
                            int64_t M, int64_t N, int64_t K, int act,
                            void *workspace, size_t ws_bytes,
                            w8a8_stream_t stream);

/* ---- a layer whose output feeds the next W8A8 layer ---------------------------
 * Source: "Issue 5 probe ...", Kernel isolation (the DiT MLP pair: the
 * up-projection img_mlp.proj feeds img_mlp.out) and Round two (step 1, the
 * dynamic per-token quantisation, applied to the next layer's input).  The
 * next layer's quantisation of this layer's output, fused with this layer:
 * the results equal, bit for bit, w8a8_linear_act(..., y, ...) followed by
 * w8a8_quant_act(y, M, N, N, q_next, a_scale_next).  The next layer then runs
 * w8a8_scaled_mm(q_next, a_scale_next, ...) on them.
 * How: the GEMM walks its output tiles row block by row block; its epilogue
 * folds every row's largest output magnitude while it stores y and reports
 * each 128-row block once its stores are complete, and the GEMM's own warps
 * (an otherwise idle warp throughout, the epilogue warps between their
 * tiles and after their last) quantise each block as it completes, reading
 * the rows back from L2, so that no separate pass over y follows the layer.
 * Two launches on `stream`, as w8a8_linear_act (for M <= 16: the layer, then
 * the quantisation kernel on y).
 *   x, ldx, packed_w, w_scale, bias, y, M, N, K, act: as w8a8_linear_act
 *   q_next       device, int8 [M, N] dense (output): the codes of y
 *   a_scale_next device, fp32 [M] (output): their per-row scales
 *   workspace    device, ws_bytes >= w8a8_linear_act_quant_workspace_bytes(M,
 *                N, K): w8a8_linear's workspace, then the row maxima and one
 *                call-tagged completion word per 128-row block (contents on
 *                entry do not matter; the last CTA of each call clears the
 *                words, so a replayed CUDA graph finds them at zero)
 * Limits as w8a8_linear, plus N % 16 == 0 (q_next is the next layer's GEMM
 * input, whose K = N) and N <= 2^28.  After a call that timed out
 * (W8A8_ERR_TIMEOUT) the words may be left set: capture CUDA graphs of this
 * call again (a new capture draws a new tag) before replaying them. */
w8a8_status w8a8_linear_act_quant_workspace_bytes(int64_t M, int64_t N, int64_t K,
                                                  size_t *bytes);
w8a8_status w8a8_linear_act_quant(const void *x, int64_t ldx, const void *packed_w,
                                  const float *w_scale, const void *bias, void *y,
                                  int64_t M, int64_t N, int64_t K, int act,
                                  int8_t *q_next, float *a_scale_next, void *workspace,
                                  size_t ws_bytes, w8a8_stream_t stream);

/* ---- the whole layer without a caller-provided workspace ---------------------
 * No counterpart on the pages: an addition for callers that cannot allocate
 * device memory when they run a layer (a plugin whose host framework owns all
 * device memory and forbids cudaMalloc inside execution callbacks, or a
 * latency-critical loop that cannot afford the device-wide synchronisation of
 * cudaMalloc / cudaFree).  Same arguments, arithmetic and results as
 * w8a8_linear, minus the workspace: the codes, scales and small-M partials go
 * to one scratch array of w8a8_linear_noalloc_max_bytes() bytes (8 MiB) that
 * every GPU loading this library holds until the process exits.  Nothing is
 * allocated.  Returns W8A8_ERR_BUFFER_TOO_SMALL, launching nothing, when
 * the codes, scales and small-M partials exceed that size
 * (w8a8_linear_workspace_bytes: M * K plus 4 M bytes, each rounded up to 256,
 * plus for M <= 16 the small-M kernel's partials).  The first call on each
 * device looks up the array's device address in the current CUDA context
 * (make it before any stream capture); the address is looked up again when
 * a call finds another context current (after a device reset, or under a
 * context the caller pushed).  All calls on a device share the array: calls
 * that overlap on the GPU (different streams without ordering) race and
 * corrupt each other. */
size_t w8a8_linear_noalloc_max_bytes(void);
w8a8_status w8a8_linear_noalloc(const void *x, int64_t ldx, const void *packed_w,
                                const float *w_scale, const void *bias, void *y,
                                int64_t M, int64_t N, int64_t K,
                                w8a8_stream_t stream);

/* ---- path selection (tests and benchmarks) ---------------------------------
 * 0 = automatic (default); 1 = always the persistent large-M GEMM (automatic
 * tile width); 2 = the small-M weight-streaming kernel (M <= 16 only, else
 * W8A8_ERR_INVALID_ARG); 3 / 4 = the 1-SM large-M GEMM with 128- / 256-wide
 * output tiles; 5 = the 2-SM (CTA pair) GEMM with 256 x 256 tiles; 7 = the
 * 2-SM GEMM with 256 x 128 tiles.  6 (and anything above 7) is not a path:
 * W8A8_ERR_INVALID_ARG.  Each path is also chosen automatically, by shape.
 * Process-wide; not synchronised with concurrent calls. */
w8a8_status w8a8_set_path(int path);

/* Name of the GEMM kernel w8a8_scaled_mm / w8a8_linear would run for this
 * shape under the current path setting (static string, for reports). */
const char *w8a8_gemm_kernel_name(int64_t M, int64_t N, int64_t K);

/* ---- harness kernel: GELU (tanh form), bf16 -> bf16 ------------------------
 * Not on the pages; it joins the up and down projections of the DiT MLP
 * workload.  y = 0.5 x (1 + tanh(sqrt(2/pi)(x + 0.044715 x^3))) in fp32,
 * rounded to bf16.  x, y device bf16 [n]; y may alias x. */
w8a8_status w8a8_gelu_tanh(const void *x, void *y, int64_t n,
                           w8a8_stream_t stream);

/* ---- errors ----------------------------------------------------------------
 * Synchronises `stream`, then returns and clears the device status word of
 * the current device: W8A8_ERR_TIMEOUT if any kernel gave up on a wait since
 * the last poll, W8A8_ERR_CUDA on an asynchronous CUDA error, else W8A8_OK.
 * After W8A8_ERR_TIMEOUT the outputs of the calls since the last poll are
 * invalid, and the call-tagged words in their workspaces (the small-M
 * kernel's slab counters, the fused next-layer quantisation's block words)
 * may be left mid-count.  A direct call draws a new tag and ignores them; a
 * captured CUDA graph replays its calls with the tags it was captured with,
 * so capture it again before replaying it. */
w8a8_status w8a8_poll_status(w8a8_stream_t stream);

/* Self-test of the bounded-wait path: launches one block that waits on a
 * barrier nothing will ever complete, with a limit of timeout_ns
 * nanoseconds (clamped to [1e3, 5e9]); the wait gives up, records
 * W8A8_ERR_TIMEOUT in the status word and the kernel exits normally. */
w8a8_status w8a8_selftest_wait_timeout(int64_t timeout_ns,
                                       w8a8_stream_t stream);

/* Self-test of the int8 tensor-core rate with no memory traffic (no
 * counterpart on the pages; the ceiling against which the GEMM kernels'
 * rates can be read): one CTA per SM issues `iters` (1 ... 2e5) groups of
 * four tcgen05.mma.kind::i8 of M = 128, N = 256, K = 32 from shared memory
 * into TMEM; the launch is timed with CUDA events on `stream` after a
 * warm-up launch.  Synchronises the stream.  *tops: int8 TOPS (2 operations
 * a multiply-add) over all SMs.  W8A8_ERR_INVALID_ARG for a null tops or
 * iters out of range; a device-side wait that gave up shows in
 * w8a8_poll_status. */
w8a8_status w8a8_selftest_int8_mma_rate(int64_t iters, w8a8_stream_t stream,
                                        double *tops);

/* Number of kernels this library has launched in this process (all devices). */
int64_t w8a8_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* W8A8_H_ */
