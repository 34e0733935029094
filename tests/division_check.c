/* division_check.c -- host proof of the fused pass's short reciprocal and quotient
 * (test infrastructure).
 *
 * The fused kernel needs two correctly rounded binary32 results per NF4 block: r = fl(1/a)
 * for the normalisation and q = fl(a/s) for the 8-bit DQ code rint(fl(q * 255)), where a is
 * the block's absmax and s the DQ block's maximum -- both 16-bit values widened to binary32.
 * It computes them with Newton-Raphson corrections on a fused multiply-add (the method whose
 * exactness conditions P. Markstein gave, IBM J. Res. Develop. 34(1), 1990):
 *
 *   reciprocal: y0 = any binary32 within 1 ulp of 1/a (the documented bound of the hardware
 *               approximation), e = fma(-a, y0, 1), r = fma(e, y0, y0);
 *   quotient:   y = fl(1/s) (the reciprocal above), q0 = fl(a * y),
 *               then once: rem = fma(-q0, s, a), q = fma(rem, y, q0).
 *
 * This program replays that arithmetic with C's fmaf (round to nearest, no contraction) and
 * compares it with the correctly rounded IEEE results 1.0f / a and a / s, for EVERY 16-bit
 * value the kernel's fast path can meet (2^-40 <= a <= 2^40), in both formats:
 *   part R: every a, every candidate y0 within 1 ulp of 1/a;
 *   part Q: every s in the fast range against every 16-bit a with 0 <= a <= s (also blocks
 *           outside the fast range: zero, subnormal or tiny a).  The DQ code
 *           rint(fl(q * 255)) must match always, the quotient itself wherever
 *           a / s >= 2^-30 (a code above 0 needs a / s >= 1/510; below 2^-30 a subnormal a
 *           may move the last bit of a quotient whose code is 0 either way).
 *
 * An optional argument sets the number of quotient corrections (default 1); 0 is the planted
 * mistake the test uses to show that the check can fail.
 * Output: "recips N bad M quotients P bad Q".  Exit status 0 iff M == 0 and Q == 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* binary32 value of a bfloat16 / binary16 bit pattern (positive patterns only) */
static float bf16_value(uint32_t h) { return from_bits(h << 16); }
static float f16_value(uint32_t h) {
  const uint32_t e = (h >> 10) & 31, m = h & 1023;
  if (e == 0) return ldexpf((float)m, -24);
  if (e == 31) return m ? NAN : INFINITY;
  return ldexpf((float)(m | 1024), (int)e - 25);
}

static float recip(float a, float y0) {
  const float e = fmaf(-a, y0, 1.0f);
  return fmaf(e, y0, y0);
}

static int corrections = 1;

static float quotient(float a, float s, float y) {
  float q = a * y;
  for (int i = 0; i < corrections; ++i) {
    const float rem = fmaf(-q, s, a);
    q = fmaf(rem, y, q);
  }
  return q;
}

static unsigned dq_code(float q) { return (unsigned)rintf(q * 255.0f); }

static long recips, bad_recips, quots, bad_quots;

static void check_recip(float a) {
  const double exact = 1.0 / (double)a;
  const float rn = 1.0f / a;
  int ex;
  frexp(exact, &ex);
  const double ulp = ldexp(1.0, ex - 24);  /* ulp of the binade of 1/a */
  for (int k = -3; k <= 3; ++k) {
    const float y0 = from_bits(to_bits(rn) + (uint32_t)k);
    if (fabs((double)y0 - exact) > ulp) continue;  /* outside the hardware bound */
    ++recips;
    if (to_bits(recip(a, y0)) != to_bits(rn)) {
      if (bad_recips < 8) fprintf(stderr, "recip mismatch a=%a y0=%a\n", a, y0);
      ++bad_recips;
    }
  }
}

static void check_format(float (*value)(uint32_t)) {
  /* the finite non-negative patterns of the format, ascending (positive patterns order like
     their values) */
  static float v[65536];
  int n = 0;
  for (uint32_t h = 0; h < 0x8000u; ++h) {
    const float x = value(h);
    if (isfinite(x)) v[n++] = x;
  }
  for (int i = 0; i < n; ++i)
    if (v[i] >= 0x1p-40f && v[i] <= 0x1p40f) check_recip(v[i]);
  for (int j = 0; j < n; ++j) {
    const float s = v[j];
    if (s < 0x1p-40f || s > 0x1p40f) continue;
    const float y = 1.0f / s;
    for (int i = 0; i <= j; ++i) {
      const float a = v[i];
      const float q = quotient(a, s, y), ref = a / s;
      ++quots;
      if ((ref >= 0x1p-30f && to_bits(q) != to_bits(ref)) || dq_code(q) != dq_code(ref)) {
        if (bad_quots < 8) fprintf(stderr, "quotient mismatch a=%a s=%a q=%a ref=%a\n", a, s, q, ref);
        ++bad_quots;
      }
    }
  }
}

int main(int argc, char** argv) {
  if (argc > 1) corrections = atoi(argv[1]);
  check_format(bf16_value);
  check_format(f16_value);
  printf("recips %ld bad %ld quotients %ld bad %ld\n", recips, bad_recips, quots, bad_quots);
  return (bad_recips == 0 && bad_quots == 0) ? 0 : 1;
}
