/* Checks, in plain C on the host, the arithmetic identity the GPU quantizer
 * uses in place of one IEEE division per element (Markstein's correction,
 * P. Markstein, IBM J. Res. Develop. 34(1), 1990):
 *
 *   r = fl32(1/s), q0 = fl32(x*r), e = fl32(x - q0*s) (fused), q1 = fl32(q0 + e*r) (fused)
 *
 * against the definition's fl32(x/s), for the per-row scales the quantizer
 * forms, s = fl32(amax/cmax) with cmax = 127 (int8) or 448 (E4M3), on rows
 * whose scale is at least 2^-100:
 *   - bf16 rows: every bf16 value |x| <= amax, both signs, for every
 *     `step`-th positive bf16 amax (step 1 is exhaustive);
 *   - fp32 rows: values planted at and a few ulps around every
 *     half-integer quotient, for pseudo-random fp32 amax.
 * int8: rne(q1) must equal rne(x/s) (the code), which here means q1 == x/s
 * wherever |x/s| >= 0.25.  E4M3: q1 with x's sign must equal x/s bit for bit
 * where |x/s| >= 2^-12, and stay below 2^-11 with x's sign elsewhere (where
 * the E4M3 code is a signed zero either way).
 * Prints the counts and exits 1 on any mismatch.  Test code only: nothing
 * here is used by the library or the oracle. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float corrected(float x, float s, float r) {
  const float q0 = x * r;
  const float e = fmaf(-q0, s, x);
  return fmaf(e, r, q0);
}

/* 0 if q1 stands in for x/s under the code's rule, else 1. */
static int bad(float x, float s, float r, int e4m3) {
  const float q = x / s;
  float q1 = corrected(x, s, r);
  if (!e4m3) return fabsf(q) >= 0.25f ? f2u(q1) != f2u(q) : (fabsf(q1) >= 0.5f);
  q1 = copysignf(q1, x);
  if (fabsf(q) >= 0x1p-12f) return f2u(q1) != f2u(q);
  return !(fabsf(q1) < 0x1p-11f && signbit(q1) == signbit(q));
}

int main(int argc, char** argv) {
  const int step = argc > 1 ? atoi(argv[1]) : 1;
  const int fp32_rows = argc > 2 ? atoi(argv[2]) : 0;
  long checked = 0, mismatches = 0;
  for (int e4m3 = 0; e4m3 < 2; ++e4m3) {
    const float cmax = e4m3 ? 448.0f : 127.0f;
    for (uint32_t ab = 1; ab < 0x7F80u; ab += (uint32_t)step) {
      const float amax = u2f(ab << 16);
      const float s = amax / cmax;
      const float r = 1.0f / s;
      if (!(s >= 0x1p-100f) || !isfinite(r)) continue;
      for (uint32_t xb = 0; xb <= ab; ++xb) {
        for (int sg = 0; sg < 2; ++sg) {
          const float x = u2f((xb << 16) | (sg ? 0x80000000u : 0u));
          ++checked;
          if (bad(x, s, r, e4m3)) {
            if (mismatches < 5) printf("mismatch: cmax %g amax %a x %a\n", cmax, amax, x);
            ++mismatches;
          }
        }
      }
    }
    uint64_t state = 0x9E3779B97F4A7C15ull;
    for (int it = 0; it < fp32_rows; ++it) {
      state = state * 6364136223846793005ull + 1442695040888963407ull;
      const uint32_t ab = (uint32_t)(state >> 33) % (0x7F000000u - 0x0C800000u) + 0x0C800000u;
      const float amax = u2f(ab);
      const float s = amax / cmax;
      const float r = 1.0f / s;
      if (!(s >= 0x1p-100f) || !isfinite(r)) continue;
      const int kmax = e4m3 ? 896 : 254;
      for (int k = -kmax; k <= kmax; ++k) {
        const float x0 = 0.5f * (float)k * s;
        for (int d = -3; d <= 3; ++d) {
          const float x = u2f((uint32_t)((int32_t)f2u(x0) + (x0 != 0.0f ? d : 0)));
          if (!(fabsf(x) <= amax)) continue;
          ++checked;
          if (bad(x, s, r, e4m3)) {
            if (mismatches < 5) printf("mismatch: cmax %g amax %a x %a\n", cmax, amax, x);
            ++mismatches;
          }
        }
      }
    }
  }
  printf("checked %ld, mismatches %ld\n", checked, mismatches);
  return mismatches != 0;
}
