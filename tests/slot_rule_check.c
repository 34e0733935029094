/* slot_rule_check.c -- host check of the fused pass's code lookup (test infrastructure).
 *
 * The fused kernel does not count midpoints.  Its rule, stated on the normalised value v:
 *   s = fma(v*v, b, a),  k = round(fma(v, s, 2^23 + 8)) - 2^23,
 *   code = k - 1 + (fl(slot_mid[k] - v) < 0),  level = slot_level[code + 1].
 * Part A replays exactly that arithmetic (fmaf, no contraction) for many binary32 values v.
 * Part B does the same for the values the kernel meets: v = fl(x fl(1/m)) for every 16-bit
 * weight x with |x| <= m of a block with maximum m (2^-40 <= m <= 2^40, the kernel's fast
 * path), for a spread of block maxima m, in both formats.
 * Both compare the code with the plain definition, the number of codebook midpoints below v
 * ("QLoRA", "How It Works": a value maps to its nearest NF4 level), and the level with the
 * codebook's level[code].
 *
 * Input (stdin, whitespace separated): a b, slot_mid[32] and slot_level[32] as hex bit
 * patterns, then the reference mids[15] and levels[16] as hex bit patterns.
 * Output: "checked N mismatches M".  Exit status 0 iff M == 0.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float a_, b_, slot_mid[32], slot_level[32], mids[15], levels[16];
static long checked, bad;

static void check(float v) {
  const float t = fmaf(v, fmaf(v * v, b_, a_), 8388616.0f);
  const uint32_t k = to_bits(t) - 0x4B000000u;
  int ref = 0;
  for (int j = 0; j < 15; ++j) ref += v > mids[j];
  ++checked;
  if (k > 31) { ++bad; return; }
  const int code = (int)k - 1 + (int)(to_bits(slot_mid[k] - v) >> 31);
  if (code != ref || to_bits(slot_level[(code + 1) & 31]) != to_bits(levels[ref])) {
    if (bad < 8) fprintf(stderr, "mismatch at v=%a: k=%u code=%d ref=%d\n", v, k, code, ref);
    ++bad;
  }
}

/* one weight x of a block with maximum m, normalised as the kernel does */
static void check_weight(float x, float m) { check(x * (1.0f / m)); }

static float bf16_value(uint32_t h) { return from_bits(h << 16); }

static float f16_value(uint32_t h) {
  const uint32_t sign = (h >> 15) & 1, e = (h >> 10) & 31, f = h & 1023;
  float mag;
  if (e == 0) mag = ldexpf((float)f, -24);
  else if (e == 31) mag = f ? NAN : INFINITY;
  else mag = ldexpf((float)(f | 1024), (int)e - 25);
  return sign ? -mag : mag;
}

/* every 16-bit x with |x| <= m, for block maxima m taken every `step` patterns */
static void weights_of_format(float (*value)(uint32_t), uint32_t step) {
  for (uint32_t hm = 0; hm < 0x8000u; hm += step) {
    const float m = value(hm);
    if (!(m >= 0x1p-40f && m <= 0x1p40f)) continue;
    for (uint32_t hx = 0; hx < 0x10000u; ++hx) {
      const float x = value(hx);
      if (fabsf(x) <= m) check_weight(x, m);
    }
  }
}

/* every binary32 within `radius` ulps of x, both signs of the step handled by bit order */
static void around(float x, uint32_t radius) {
  const uint32_t mag = to_bits(fabsf(x)), sign = to_bits(x) & 0x80000000u;
  const uint32_t lo = mag > radius ? mag - radius : 0, hi = mag + radius;
  for (uint32_t m = lo; m <= hi; ++m) check(from_bits(m | sign));
}

static int read_hex(uint32_t* u) { unsigned x; if (scanf("%x", &x) != 1) return 0; *u = x; return 1; }

int main(void) {
  uint32_t u;
  float* dst[] = {&a_, &b_};
  for (int i = 0; i < 2; ++i) { if (!read_hex(&u)) return 2; *dst[i] = from_bits(u); }
  for (int i = 0; i < 32; ++i) { if (!read_hex(&u)) return 2; slot_mid[i] = from_bits(u); }
  for (int i = 0; i < 32; ++i) { if (!read_hex(&u)) return 2; slot_level[i] = from_bits(u); }
  for (int i = 0; i < 15; ++i) { if (!read_hex(&u)) return 2; mids[i] = from_bits(u); }
  for (int i = 0; i < 16; ++i) { if (!read_hex(&u)) return 2; levels[i] = from_bits(u); }

  const uint32_t top = to_bits(1.0f + 0x1p-20f);
  /* 1. a prime-strided sweep of every magnitude up to 1 + 2^-20, both signs */
  for (uint32_t m = 0; m <= top; m += 61) { check(from_bits(m)); check(from_bits(m | 0x80000000u)); }
  /* 2. the neighbourhood of every midpoint: where the code changes */
  for (int j = 0; j < 15; ++j) around(mids[j], 1u << 18);
  /* 3. the neighbourhood of every slot boundary: h(v) = a v + b v^3 + 8.5 crossing an
        integer n, located by bisection in binary64 on each monotone piece */
  const double a = a_, b = b_;
  const double crit = (b < 0 && a > 0) ? sqrt(a / (-3.0 * b)) : 2.0;
  const double cuts[4] = {-1.0 - 0x1p-20, -fmin(crit, 1.0 + 0x1p-20), fmin(crit, 1.0 + 0x1p-20),
                          1.0 + 0x1p-20};
  for (int piece = 0; piece < 3; ++piece) {
    double lo = cuts[piece], hi = cuts[piece + 1];
    if (!(hi > lo)) continue;
    for (int n = 0; n <= 17; ++n) {
      double x0 = lo, x1 = hi, f0 = a * x0 + b * x0 * x0 * x0 + 8.5 - n,
             f1 = a * x1 + b * x1 * x1 * x1 + 8.5 - n;
      if ((f0 < 0) == (f1 < 0)) continue;
      for (int it = 0; it < 200; ++it) {
        double xm = 0.5 * (x0 + x1), fm = a * xm + b * xm * xm * xm + 8.5 - n;
        if ((fm < 0) == (f0 < 0)) { x0 = xm; f0 = fm; } else { x1 = xm; }
      }
      around((float)x0, 1u << 18);
    }
  }
  /* 4. the kernel's form: 16-bit weights against block maxima, both formats */
  weights_of_format(bf16_value, 13);
  weights_of_format(f16_value, 29);
  /* 5. special values */
  const float special[] = {0.0f, -0.0f, 1.0f, -1.0f, 0x1p-149f, -0x1p-149f, 0x1p-126f,
                           1.0f + 0x1p-20f, -1.0f - 0x1p-20f};
  for (unsigned i = 0; i < sizeof special / sizeof special[0]; ++i) check(special[i]);
  printf("checked %ld mismatches %ld\n", checked, bad);
  return bad != 0;
}
