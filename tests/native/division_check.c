/*
 * Host check of the quantize kernel's division-free encode step.
 *
 * The kernel forms v = RN(w / a) for |w| <= a as
 *     y  = RN(1 / a)                      (correctly rounded reciprocal)
 *     q  = RN(w * y)
 *     v' = RN(RN(w - a q) * y + q)        (two fused multiply-adds)
 * which is Markstein's correction step for a correctly rounded quotient.  The
 * step is exact when the remainder w - a q is representable: its lowest bit
 * is ulp(a) ulp(q) = 2^(ea + eq - 46), which must not fall below the
 * smallest subnormal 2^-149, so ea + eq >= -103.  Only quotients with
 * |v| >= 2^-5 can decide a code (every NF4 decision threshold is at least
 * 0.0398 from zero), i.e. eq >= -5, so the kernel keeps the step for
 * 2^-98 <= a < 2^120 and divides elsewhere.
 *
 * This program runs the same three steps with C's IEEE float operations and
 * the C library's fmaf (one rounding, as the GPU's FMA) over that range of a
 * and checks, per pair:
 *   |w / a| >= 2^-5 : v' is the IEEE quotient w / a bit for bit;
 *   otherwise        : v' and w / a are both below 0.039 in magnitude, so
 *                      both encode to the zero level.
 * It counts the pairs where that fails.
 * Build: gcc -O2 -ffp-contract=off -o division_check division_check.c -lm
 * Usage: division_check <n_scales> <n_per_scale> <seed>
 * Prints "pairs mismatches" on one line; exit status 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint64_t rng_state;
/* splitmix64: a small counter-based generator */
static uint64_t next_u64(void) {
  uint64_t z = (rng_state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static float from_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}
static uint32_t to_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* 1 when the kernel's quotient decides the same code as the IEEE one */
static int corrected_ok(float w, float a) {
  const float y = 1.0f / a;
  const float q = w * y;
  const float v = fmaf(fmaf(-a, q, w), y, q);
  const float ref = w / a;
  if (fabsf(ref) >= 0x1p-5f) return to_bits(v) == to_bits(ref);
  return fabsf(v) < 0.039f && fabsf(ref) < 0.039f;
}

int main(int argc, char** argv) {
  const long n_scales = argc > 1 ? atol(argv[1]) : 1000;
  const long per = argc > 2 ? atol(argv[2]) : 10000;
  rng_state = argc > 3 ? strtoull(argv[3], NULL, 10) : 1;
  long long pairs = 0, bad = 0;
  for (long s = 0; s < n_scales; ++s) {
    /* a: any significand, exponent across the kernel's fast range (biased
     * exponents 29 .. 246 are 2^-98 .. 2^119), the two ends included, and
     * a third of the scales in the lowest 16 binades of the range */
    uint32_t e = 29 + (uint32_t)(next_u64() % 218);
    if (s % 3 == 0) e = 29 + (uint32_t)(next_u64() % 16);
    if (s == 0) e = 29;
    if (s == 1) e = 246;
    const uint32_t mant = (uint32_t)(next_u64() & 0x7fffffu);
    const float a = from_bits((e << 23) | mant);
    /* w: the block's max itself and its neighbours, then |w| <= a with a
     * uniform significand and an exponent 0 .. 40 below a's (subnormal w
     * included), both signs */
    float edge[4] = {a, -a, nextafterf(a, 0.0f), -nextafterf(a, 0.0f)};
    for (int i = 0; i < 4; ++i) {
      pairs++;
      bad += !corrected_ok(edge[i], a);
    }
    for (long i = 0; i < per; ++i) {
      const uint64_t r = next_u64();
      const uint32_t de = (uint32_t)(r % 41);
      const uint32_t wm = (uint32_t)((r >> 8) & 0x7fffffu);
      const uint32_t we = e >= de ? e - de : 0;
      float w = from_bits((we << 23) | wm);
      if (fabsf(w) > a) w = a;
      if ((r >> 40) & 1) w = -w;
      pairs++;
      bad += !corrected_ok(w, a);
    }
  }
  printf("%lld %lld\n", pairs, bad);
  return 0;
}
