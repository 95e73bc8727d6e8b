/* Exhaustive check behind the quantisation kernels' code arithmetic.
 *
 * The kernels form the code of x as rint(q1), q1 the one-step reciprocal
 * refinement of x / s: q0 = RN(x * inv), r0 = x - s * q0 (one FMA, exact),
 * q1 = RN(q0 + r0 * inv) (one FMA), inv = RN(1 / s).  The method defines the
 * code as rint(RN(x / s)) (IEEE division), with s = RN(amax / 127).  This
 * program visits every positive finite bf16 amax whose s is at least 1e-30
 * (smaller scales take the IEEE quotient in the kernels) and every bf16 x in
 * [0, amax], and counts the pairs where the two codes differ.  It also counts
 * the differences without the refinement step (q0 alone), to show the step
 * is needed, and spot-checks negative x (every operation is odd in x).
 *
 * Prints: pairs <n> one_step <mismatches> no_step <mismatches> negative <mismatches>
 * Build: gcc -O2 -fopenmp -ffp-contract=off (no contraction, IEEE float). */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bf16_value(uint32_t h) {
  const uint32_t u = h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

int main(void) {
  long long pairs = 0, one_step = 0, no_step = 0, negative = 0;
  for (uint32_t ha = 1; ha < 0x7F80u; ++ha) { /* positive finite bf16 */
    const float amax = bf16_value(ha);
    const float s = amax / 127.0f;
    if (!(s >= 1e-30f)) continue;
    const float inv = 1.0f / s;
    long long d1 = 0, d0 = 0, dn = 0;
#pragma omp parallel for reduction(+ : d1, d0, dn) schedule(static)
    for (uint32_t hx = 0; hx <= ha; ++hx) { /* bf16 bit patterns are ordered for x >= 0 */
      const float x = bf16_value(hx);
      const float code = nearbyintf(x / s);
      const float q0 = x * inv;
      const float r0 = fmaf(-s, q0, x);
      const float q1 = fmaf(r0, inv, q0);
      d1 += nearbyintf(q1) != code;
      d0 += nearbyintf(q0) != code;
      if ((hx & 0x3Fu) == 0x15u) {
        const float xn = -x;
        const float p0 = xn * inv, e0 = fmaf(-s, p0, xn), p1 = fmaf(e0, inv, p0);
        dn += nearbyintf(p1) != nearbyintf(xn / s);
      }
    }
    pairs += (long long)ha + 1;
    one_step += d1;
    no_step += d0;
    negative += dn;
  }
  printf("pairs %lld one_step %lld no_step %lld negative %lld\n", pairs, one_step, no_step,
         negative);
  return 0;
}
