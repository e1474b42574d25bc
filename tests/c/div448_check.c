/* The fp8 group scale's division amax / 448, as the device computes it for
 * 2^-120 <= amax <= FLT_MAX (div448_rn in the library's device code: the
 * product by c = RN(1/448), corrected once by its exact remainder with fma),
 * checked against the exactly rounded quotient for every binary32 in that
 * range. The exact quotient is decided from exact residuals: q * 448 and
 * x - q * 448 are exact in binary64 for the candidates q compared, and ties go
 * to the even significand. Exit status 0 if every value matches. With the
 * argument "mutant" it checks the product without its correction step instead
 * (a plausible slip), over part of the range, and exits 0 only if that is
 * caught. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float u2f(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f2u(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float div448_formula(float x, int corrected) {
  const float c = 0x1.24924ap-9f;
  const float q0 = x * c;
  if (!corrected) return q0;
  const float r = fmaf(-q0, 448.0f, x);
  return fmaf(r, c, q0);
}

static float div448_exact(float x) {
  const float q = (float)((double)x / 448.0);
  float best = q;
  double bd = -1.0;
  for (int k = -2; k <= 2; ++k) {
    const float cand = u2f((uint32_t)((int64_t)f2u(q) + k));
    if (!(cand >= 0.0f) || isinf(cand)) continue;
    const double d = fabs((double)x - (double)cand * 448.0);
    if (bd < 0.0 || d < bd || (d == bd && (f2u(cand) & 1u) == 0u)) {
      bd = d;
      best = cand;
    }
  }
  return best;
}

int main(int argc, char** argv) {
  const int mutant = argc > 1 && strcmp(argv[1], "mutant") == 0;
  const uint32_t lo = f2u(0x1p-120f);
  const uint32_t hi = mutant ? lo + (1u << 24) : 0x7F800000u; /* exclusive */
  unsigned long long bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static, 1 << 16)
  for (int64_t u = lo; u < (int64_t)hi; ++u) {
    const float x = u2f((uint32_t)u);
    if (f2u(div448_formula(x, !mutant)) != f2u(div448_exact(x))) ++bad;
  }
  printf("%s: %llu mismatches over %u values\n", mutant ? "mutant" : "formula", bad, hi - lo);
  return mutant ? (bad == 0) : (bad != 0);
}
