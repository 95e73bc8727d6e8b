/*
 * w8a8_oracle.c -- plain CPU oracle for the W8A8 int8-dynamic linear path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file.  It may be used by the tests, by the smoke check and by the
 * CPU-baseline leg of the benchmark, and by nothing else.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (sources, by page title and section):
 *
 *  - "Issue 5 probe: int8 quantized DiT serve paths on the RTX 3090", section
 *    "Round two ... W8A8 int8-dynamic": the artifact is int8 weights with fp32
 *    per-output-channel scales plus *dynamic per-token symmetric* int8
 *    activations, served by an int8 scaled matmul (quantize the activations,
 *    multiply int8 x int8, apply the row and column scales).  Same page,
 *    "Round one": the weights are per-output-channel symmetric.
 *  - "INT8 Quant for Dual-Max Recipe": W8A8 runs int8 x int8 on the integer
 *    tensor cores with no dequantisation of the weights, and the activation
 *    quantisation is dynamic per token.
 *  - "Online Quantization", section "Parameters": activation_scheme "dynamic"
 *    means the activation scale is computed at run time.
 *
 * The pages do not spell out the rounding rules.  The readings used here
 * (each one is listed with its reason in the design notes of the repository):
 *    scale  = amax / 127 in fp32 (IEEE division, round to nearest even);
 *    q      = clamp(round_half_even(x / scale), -127, 127), IEEE fp32
 *             division, never a multiply by a reciprocal;
 *    a row whose amax is 0 gets scale 0 and q = 0;
 *    acc    = exact integer sum of q*w (checked in int64, stored as int32);
 *    y      = bf16_rne( ((float)acc * a_scale[m]) * w_scale[n] + bias[n] ),
 *             every step one fp32 operation rounded to nearest even.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fno-fast-math -shared -fPIC.
 * -ffp-contract=off keeps every multiply and add a separately rounded fp32
 * operation, as the definition above states.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_EOVERFLOW 2

/* ---- bf16 <-> fp32 ------------------------------------------------------
 * bf16 is the upper half of an IEEE binary32.  Widening is exact.  Narrowing
 * rounds to nearest, ties to even, on the 16 discarded bits. */
static float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u) {
    return (uint16_t)((u >> 16) | 0x0040u); /* quiet NaN, sign kept */
  }
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* double -> bf16, one rounding (nearest, ties even).  The double is first
 * narrowed to fp32 with round-to-odd (truncate, then force the last bit to 1
 * if anything was discarded); fp32 keeps 16 more bits than bf16, so the
 * second, nearest-even narrowing then equals a single direct rounding. */
static uint16_t f64_to_bf16_rne(double g) {
  float f = (float)g;
  if ((double)f != g && isfinite(f)) {
    if (fabs((double)f) > fabs(g)) f = nextafterf(f, 0.0f);
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    u |= 1u;
    memcpy(&f, &u, sizeof f);
  }
  return f32_to_bf16_rne(f);
}

uint16_t w8a8o_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }
uint16_t w8a8o_f64_to_bf16(double g) { return f64_to_bf16_rne(g); }
float w8a8o_bf16_to_f32(uint16_t h) { return bf16_to_f32(h); }

/* ---- step 1: dynamic per-token symmetric activation quantisation --------
 * x: bf16 [M, K] with row stride ldx (elements).  q: int8 [M, K] dense.
 * a_scale: fp32 [M]. */
int w8a8o_quant_act(const uint16_t *x, int64_t M, int64_t K, int64_t ldx,
                    int8_t *q, float *a_scale) {
  if (!x || !q || !a_scale || M < 0 || K < 0 || ldx < K) return ORACLE_EINVAL;
  int64_t m;
#pragma omp parallel for schedule(static)
  for (m = 0; m < M; ++m) {
    const uint16_t *xr = x + m * ldx;
    int8_t *qr = q + m * K;
    /* amax over the row */
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = fabsf(bf16_to_f32(xr[k]));
      if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
      a_scale[m] = 0.0f;
      for (int64_t k = 0; k < K; ++k) qr[k] = 0;
      continue;
    }
    float s = amax / 127.0f;
    a_scale[m] = s;
    for (int64_t k = 0; k < K; ++k) {
      float v = bf16_to_f32(xr[k]) / s; /* IEEE fp32 division */
      float r = nearbyintf(v);          /* default mode: nearest, ties even */
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      qr[k] = (int8_t)r;
    }
  }
  return ORACLE_OK;
}

/* ---- step 2: int8 x int8 -> int32 GEMM -----------------------------------
 * acc[m, n] = sum_k q[m, k] * w[n, k].  q: [M, K], w: [N, K] (K contiguous),
 * acc: [M, N].  The sum is formed in int64 and must fit in int32; if any
 * element does not, ORACLE_EOVERFLOW is returned (and that element is left
 * as the truncated value, which callers must not use). */
int w8a8o_gemm_i32(const int8_t *q, const int8_t *w, int64_t M, int64_t N,
                   int64_t K, int32_t *acc) {
  if (!q || !w || !acc || M < 0 || N < 0 || K < 0) return ORACLE_EINVAL;
  int overflow = 0;
  int64_t m;
#pragma omp parallel for schedule(static) reduction(| : overflow)
  for (m = 0; m < M; ++m) {
    const int8_t *qr = q + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const int8_t *wr = w + n * K;
      int64_t s = 0;
      for (int64_t k = 0; k < K; ++k) s += (int64_t)qr[k] * (int64_t)wr[k];
      if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
      acc[m * N + n] = (int32_t)s;
    }
  }
  return overflow ? ORACLE_EOVERFLOW : ORACLE_OK;
}

/* ---- step 3: dequantising epilogue ---------------------------------------
 * y[m, n] = bf16_rne(((float)acc[m, n] * a_scale[m]) * w_scale[n] + bias[n]).
 * bias may be NULL (then the add is skipped, not "+0"). */
static uint16_t epilogue_one(int32_t acc, float as, float ws,
                             const uint16_t *bias, int64_t n) {
  float t = (float)acc; /* int32 -> fp32, nearest even */
  t = t * as;
  t = t * ws;
  if (bias) t = t + bf16_to_f32(bias[n]);
  return f32_to_bf16_rne(t);
}

int w8a8o_epilogue(const int32_t *acc, const float *a_scale,
                   const float *w_scale, const uint16_t *bias, int64_t M,
                   int64_t N, uint16_t *y) {
  if (!acc || !a_scale || !w_scale || !y || M < 0 || N < 0)
    return ORACLE_EINVAL;
  int64_t m;
#pragma omp parallel for schedule(static)
  for (m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n)
      y[m * N + n] = epilogue_one(acc[m * N + n], a_scale[m], w_scale[n], bias, n);
  return ORACLE_OK;
}

/* ---- the whole layer ------------------------------------------------------
 * y = epilogue(gemm(quant(x), w)).  q_out / a_scale_out / acc_out receive
 * the intermediate results when not NULL. */
int w8a8o_linear(const uint16_t *x, int64_t ldx, const int8_t *w,
                 const float *w_scale, const uint16_t *bias, int64_t M,
                 int64_t N, int64_t K, uint16_t *y, int8_t *q_out,
                 float *a_scale_out, int32_t *acc_out) {
  if (!x || !w || !w_scale || !y || M < 0 || N < 0 || K < 0)
    return ORACLE_EINVAL;
  int8_t *q = q_out ? q_out : (int8_t *)malloc((size_t)(M * K) + 1);
  float *as = a_scale_out ? a_scale_out : (float *)malloc(sizeof(float) * (size_t)M + 4);
  int32_t *acc = acc_out ? acc_out : (int32_t *)malloc(sizeof(int32_t) * (size_t)(M * N) + 4);
  int rc = ORACLE_EINVAL;
  if (q && as && acc) {
    rc = w8a8o_quant_act(x, M, K, ldx, q, as);
    if (rc == ORACLE_OK) rc = w8a8o_gemm_i32(q, w, M, N, K, acc);
    if (rc == ORACLE_OK) rc = w8a8o_epilogue(acc, as, w_scale, bias, M, N, y);
  }
  if (!q_out) free(q);
  if (!a_scale_out) free(as);
  if (!acc_out) free(acc);
  return rc;
}

/* ---- sampled outputs at full size ------------------------------------------
 * For count pairs (rows[i], cols[i]): acc and y of that one output, from the
 * already quantised activations.  Used where the full product is too large to
 * form on the CPU in a test. */
int w8a8o_sampled(const int8_t *q, const float *a_scale, const int8_t *w,
                  const float *w_scale, const uint16_t *bias, int64_t K,
                  const int64_t *rows, const int64_t *cols, int64_t count,
                  int32_t *acc_out, uint16_t *y_out) {
  if (!q || !a_scale || !w || !w_scale || !rows || !cols || count < 0)
    return ORACLE_EINVAL;
  int overflow = 0;
  int64_t i;
#pragma omp parallel for schedule(static) reduction(| : overflow)
  for (i = 0; i < count; ++i) {
    const int8_t *qr = q + rows[i] * K;
    const int8_t *wr = w + cols[i] * K;
    int64_t s = 0;
    for (int64_t k = 0; k < K; ++k) s += (int64_t)qr[k] * (int64_t)wr[k];
    if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
    if (acc_out) acc_out[i] = (int32_t)s;
    if (y_out)
      y_out[i] = epilogue_one((int32_t)s, a_scale[rows[i]], w_scale[cols[i]], bias, cols[i]);
  }
  return overflow ? ORACLE_EOVERFLOW : ORACLE_OK;
}

/* ---- load-time weight repack --------------------------------------------
 * The pages name the step (weights are transposed and repacked once as they
 * are loaded, then applied: Round two, kernel-path verification) but not a
 * layout; the layout is this library's
 * own and is defined here from its written description, independently of the
 * CUDA code:
 *
 *   Np = N rounded up to 256, Kp = K rounded up to 128.
 *   The packed buffer is an array of tiles T(nb, kb), nb < Np/128,
 *   kb < Kp/128, tile T(nb, kb) at byte (nb * (Kp/128) + kb) * 16384.
 *   Inside a tile, weight row r = n - 128*nb (0..127) and byte c = k - 128*kb
 *   (0..127) sit at
 *       r*128 + (((c / 16) XOR (r % 8)) * 16) + (c % 16)
 *   i.e. each 128-byte row of K is cut into eight 16-byte chunks and chunk j
 *   of row r is stored at chunk position j XOR (r mod 8).  Entries with
 *   n >= N or k >= K are zero.
 */
int w8a8o_pack_weight(const int8_t *w, int64_t N, int64_t K, int8_t *packed) {
  if (!w || !packed || N < 0 || K < 0) return ORACLE_EINVAL;
  int64_t Np = (N + 255) / 256 * 256;
  int64_t Kp = (K + 127) / 128 * 128;
  int64_t kblocks = Kp / 128;
  memset(packed, 0, (size_t)(Np * Kp));
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t k = 0; k < K; ++k) {
      int64_t nb = n / 128, r = n % 128;
      int64_t kb = k / 128, c = k % 128;
      int64_t tile = (nb * kblocks + kb) * 16384;
      int64_t off = r * 128 + (((c / 16) ^ (r % 8)) * 16) + (c % 16);
      packed[tile + off] = w[n * K + k];
    }
  }
  return ORACLE_OK;
}

int64_t w8a8o_packed_bytes(int64_t N, int64_t K) {
  return ((N + 255) / 256 * 256) * ((K + 127) / 128 * 128);
}

/* ---- GELU (tanh form), bf16 -> bf16 ----------------------------------------
 * Only used between the up and down projections of the DiT MLP workload; the
 * pages do not define it.  GELU_tanh(x) = 0.5 x (1 + tanh(u)) with
 * u = sqrt(2/pi) (x + 0.044715 x^3).  Since 0.5 (1 + tanh(u)) = 1 / (1 + e^(-2u))
 * exactly, it is evaluated in double as x * sigma(2u), with sigma written so
 * that no step cancels (1 + tanh(u) loses every digit once tanh(u) rounds to
 * -1, e.g. u < -19 in double), then rounded once to bf16. */
int w8a8o_gelu_tanh(const uint16_t *x, int64_t n, uint16_t *y) {
  if (!x || !y || n < 0) return ORACLE_EINVAL;
  const double c = sqrt(2.0 / 3.14159265358979323846);
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < n; ++i) {
    double v = (double)bf16_to_f32(x[i]);
    double u = c * (v + 0.044715 * v * v * v);
    double e = exp(-2.0 * fabs(u));           /* in (0, 1] */
    double sig = u >= 0.0 ? 1.0 / (1.0 + e) : e / (1.0 + e);
    y[i] = f64_to_bf16_rne(v * sig);
  }
  return ORACLE_OK;
}

/* ---- online weight quantisation ------------------------------------------
 * "Online Quantization", Overview: quantised weights and scales are computed
 * while the model loads, from bf16 weights.  "Issue 5 probe ...", Round one:
 * the weights are per-output-channel symmetric.  So each output channel (a row
 * of W[N, K]) follows the rule of the activation rows: scale = amax / 127,
 * code = clamp(rne(w / scale), -127, 127), a zero row gets scale 0.
 * w: bf16 [N, K]; q: int8 [N, K]; w_scale: fp32 [N]. */
int w8a8o_quant_weight(const uint16_t *w, int64_t N, int64_t K, int8_t *q, float *w_scale) {
  return w8a8o_quant_act(w, N, K, K, q, w_scale);
}

/* ---- static (calibrated) per-tensor activation scale ------------------------
 * "Online Quantization", Parameters: activation_scheme "dynamic" selects run-
 * time activation scaling; the other scheme keeps one calibrated fp32 scale
 * for the whole tensor.  code = clamp(rne(x / scale), -127, 127); values
 * beyond the calibrated range saturate.  A scale that is not > 0 (0, negative,
 * NaN) gives codes 0 (reading: no usable scale).  a_scale_out[m] = scale (or
 * 0) so the scaled GEMM applies it per row unchanged. */
int w8a8o_quant_act_static(const uint16_t *x, int64_t M, int64_t K, int64_t ldx, float scale,
                           int8_t *q, float *a_scale_out) {
  if (!x || !q || M < 0 || K < 0 || ldx < K) return ORACLE_EINVAL;
  const int usable = scale > 0.0f; /* false for NaN too */
  int64_t m;
#pragma omp parallel for schedule(static)
  for (m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      if (!usable) {
        q[m * K + k] = 0;
        continue;
      }
      float v = bf16_to_f32(x[m * ldx + k]) / scale;
      float r = nearbyintf(v);
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      q[m * K + k] = (int8_t)r;
    }
    if (a_scale_out) a_scale_out[m] = usable ? scale : 0.0f;
  }
  return ORACLE_OK;
}

/* ---- compressed-tensors int32 weight storage -----------------------------
 * "Issue 5 probe ...", Artifact: weights stored with pack_to_int32, four
 * bytes to an int32 word, each the weight plus 128 as an unsigned byte.
 * Reading (the page gives no bit order): the
 * four consecutive K elements k = 4j .. 4j+3 of a row share int32 word j,
 * element 4j+i in bits [8i, 8i+8) as the unsigned byte (w + 128).
 * packed: int32 [N, K/4]; w: int8 [N, K]. */
int w8a8o_unpack_int32(const int32_t *packed, int64_t N, int64_t K, int8_t *w) {
  if (!packed || !w || N < 0 || K < 0 || K % 4 != 0) return ORACLE_EINVAL;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      uint32_t word = (uint32_t)packed[n * (K / 4) + k / 4];
      uint32_t byte = (word >> (8 * (k % 4))) & 0xFFu;
      w[n * K + k] = (int8_t)((int)byte - 128);
    }
  return ORACLE_OK;
}

int w8a8o_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Sets the number of threads later calls use (for single-thread timings). */
void w8a8o_set_num_threads(int n) {
#ifdef _OPENMP
  extern void omp_set_num_threads(int);
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}
