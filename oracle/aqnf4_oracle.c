/*
 * aqnf4_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, scalar CPU statement of the per-layer NF4 pass: blockwise absmax NF4
 * quantization with a 16-level normal-quantile codebook, nibble packing, double
 * quantization of the absmax constants, dequantization, the per-layer reconstruction
 * error, and top-K layer selection under a byte budget.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load this.
 * It shares no code, table or constant generator with the CUDA library; both sides
 * derive the codebook from the definition on their own.
 *
 * Built as plain C11 with -O2 -ffp-contract=off (no fused multiply-add, no fast-math):
 * every float operation below is one IEEE-754 binary32 operation rounded to nearest
 * even, every double operation one binary64 operation.
 *
 * Sources (page title, section):
 *   [QLoRA/HIW]  "QLoRA" (ai360xpert.com), "How It Works": NF4 gives each of its 16
 *                values an equal share of the weights; the per-block scales get an
 *                8-bit encoding of their own, worth about 0.37 bits per weight; a
 *                training pass computes with 16-bit values rebuilt from the storage.
 *   [QLoRA/Idea] "QLoRA" (ai360xpert.com), "The Idea": NF4 is built for normally
 *                distributed weights.
 *   [QLE/NF4]    "QLoRA Explained" (devtoolshub.net), "NF4" and "4-Bit Quantization in
 *                QLoRA": the data type follows the normal distribution of weights.
 *   [QLE/DQ]     "QLoRA Explained", "Double Quantization": the per-block
 *                constants restore each block's range, and DQ stores them compressed too.
 *   [AQLoRA/abs] arxivdaily 2608.23816, "English abstract": a single sweep over the
 *                weights orders the layers by their NF4 error and holds the highest-error
 *                ones in 16 bits while a byte budget allows; the quality setting needs
 *                0.2 GiB of extra memory.
 *   [AQLoRA/TD]  "AQLoRA: A Zero-Search Recipe for Fast Quantized LoRA Fine-Tuning",
 *                "Technical Details": every layer is ranked; the budget is configurable.
 *
 * Readings where the pages are silent (each is also listed in the design notes):
 *   - levels: 8 positive quantiles at evenly spaced probabilities from 1/2 (dropped) to
 *     p_max, 7 negative ones likewise, an exact 0, all divided by the largest magnitude;
 *     default p_max = 1 - (1/32 + 1/30)/2.
 *   - midpoints m_j: the binary64 midpoint of the two neighbouring binary32 levels,
 *     rounded to binary32; code = #{ j : v > m_j } (a value on a midpoint goes down).
 *   - normalisation: v = fl(x * fl(1/a)), a = max |x| over the 64-element block; a block
 *     whose absmax is below the binary32 normal range is first scaled by 2^64 (exact),
 *     and an all-zero block codes to the exact-zero level 7.
 *   - packing: byte i = code[2i] << 4 | code[2i+1]; an odd tail leaves the low nibble 0.
 *   - reconstruction: w_hat = dtype_rn(fl(q[code] * a)); the layer score is
 *     sqrt(sum (x - w_hat)^2 / sum x^2), sums in binary64 in element order.
 *   - double quantization: per 256 constants s = max a; code8 = rint_even(fl(fl(a/s)*255)).
 *   - the DQ-absmax score (an option): the same error with w_hat reconstructed from the
 *     double-quantized constant a' = fl(fl(code8/255) * s) -- what a stored NF4 + DQ model
 *     dequantizes to -- while the codes still come from the binary32 absmax.
 *   - linear layer on NF4 weights: y = x w_hat^T in binary64, w_hat rebuilt as dequantize does.
 *   - mean-centred DQ (an option, from outside the pages): per 256 constants the binary64
 *     tree-sum mean mu, h = max |a - mu|, q = rint_even(fl(fl((a - mu)/h) * 127)) stored as
 *     q + 128, rebuilt as fl(fl(fl(q/127) * h) + mu).
 *   - selection: sort by (score desc, index asc, NaN last); keep the longest prefix with
 *     at most k_cap layers and total incremental cost <= budget.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_F16 0
#define OR_BF16 1
#define OR_BLOCK 64
#define OR_DQ_BLOCK 256

/* ------------------------------------------------------------------ formats */

static float or_bits_to_f32(uint32_t u) {
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static uint32_t or_f32_to_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
}

/* binary16 / bfloat16 bit pattern -> value (exact). */
static float or_load(uint16_t h, int dtype) {
  if (dtype == OR_BF16) return or_bits_to_f32((uint32_t)h << 16);
  /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
  int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);                /* zero or subnormal */
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + m), e - 25);    /* 1.m * 2^(e-15) */
  return (float)(sign ? -v : v);
}

/* Round x (any binary32 value, handled exactly in binary64) to the nearest value of a
   binary format with p significand bits, smallest normal exponent emin and largest
   finite value maxv; ties to even; overflow goes to infinity (IEEE 754 round to nearest). */
static double or_round_to_format(double x, int p, int emin, double maxv) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  double ax = fabs(x);
  int E;
  frexp(ax, &E); /* ax = f * 2^E, f in [0.5, 1): leading bit has weight 2^(E-1) */
  int lead = E - 1;
  if (lead < emin) lead = emin; /* subnormal range: fixed quantum */
  double quantum = ldexp(1.0, lead - (p - 1));
  double r = nearbyint(ax / quantum) * quantum; /* default rounding mode: ties to even */
  if (r > maxv) r = INFINITY;
  return x < 0 ? -r : r;
}

/* value (exactly representable in the format after or_round_to_format) -> bit pattern */
static uint16_t or_encode(double y, int dtype) {
  const int p = dtype == OR_BF16 ? 8 : 11;
  const int bias = dtype == OR_BF16 ? 127 : 15;
  const int emin = 1 - bias;
  uint16_t sign = signbit(y) ? 0x8000u : 0u;
  if (isnan(y)) return dtype == OR_BF16 ? 0x7FC0u : 0x7E00u;
  double ay = fabs(y);
  uint16_t expmask = dtype == OR_BF16 ? 0x7F80u : 0x7C00u;
  if (isinf(ay)) return sign | expmask;
  if (ay == 0.0) return sign;
  int E;
  frexp(ay, &E);
  int lead = E - 1;
  if (lead < emin) { /* subnormal: fraction counts quanta of 2^(emin-(p-1)) */
    uint16_t frac = (uint16_t)(ay / ldexp(1.0, emin - (p - 1)));
    return sign | frac;
  }
  uint16_t frac = (uint16_t)(ay / ldexp(1.0, lead - (p - 1)) - ldexp(1.0, p - 1));
  uint16_t ebits = (uint16_t)(lead + bias);
  return sign | (uint16_t)(ebits << (p - 1)) | frac;
}

static uint16_t or_round_to_dtype(float f, int dtype) {
  double y = dtype == OR_BF16 ? or_round_to_format(f, 8, -126, ldexp(255.0, 120))
                              : or_round_to_format(f, 11, -14, 65504.0);
  return or_encode(y, dtype);
}

/* ---------------------------------------------------------------- codebook */

static double or_normal_cdf(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

/* Inverse of the standard normal CDF by bisection: slow, but plainly correct to the
   resolution of binary64 because the CDF is monotone. */
static double or_normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 400; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (or_normal_cdf(mid) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

double oracle_default_pmax(void) { return 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0); }

/* NF4 levels and midpoints ([QLoRA/HIW], [QLoRA/Idea], [QLE/NF4]).
   Returns 0 on success, -1 if p_max is not in (1/2, 1). */
int oracle_codebook(double p_max, float levels[16], float mids[15]) {
  if (!(p_max > 0.5 && p_max < 1.0)) return -1;
  double q[16];
  int n = 0;
  /* 7 negative levels: probabilities p_max, ..., stepping toward 1/2 in 7 equal steps,
     the 1/2 itself (which would give 0) left out. */
  for (int k = 0; k < 7; ++k) q[n++] = -or_normal_quantile(p_max + k * (0.5 - p_max) / 7.0);
  q[n++] = 0.0;
  /* 8 positive levels: same with 8 equal steps. */
  for (int k = 0; k < 8; ++k) q[n++] = or_normal_quantile(p_max + k * (0.5 - p_max) / 8.0);
  /* sort ascending (insertion sort; 16 values) */
  for (int i = 1; i < 16; ++i)
    for (int j = i; j > 0 && q[j - 1] > q[j]; --j) {
      double t = q[j];
      q[j] = q[j - 1];
      q[j - 1] = t;
    }
  double big = 0.0;
  for (int i = 0; i < 16; ++i)
    if (fabs(q[i]) > big) big = fabs(q[i]);
  for (int i = 0; i < 16; ++i) levels[i] = (float)(q[i] / big);
  for (int j = 0; j < 15; ++j) mids[j] = (float)(((double)levels[j] + (double)levels[j + 1]) / 2.0);
  return 0;
}

/* ---------------------------------------------------------------- quantize */

static int or_code_of(float v, const float mids[15]) {
  int c = 0;
  for (int j = 0; j < 15; ++j)
    if (v > mids[j]) ++c; /* NaN compares false: code 0 */
  return c;
}

/* absmax with NaN propagation: NaN if any element is NaN, else max |x|. */
static float or_block_absmax(const uint16_t* w, int dtype, int64_t start, int len) {
  float a = 0.0f;
  for (int i = 0; i < len; ++i) {
    float ax = fabsf(or_load(w[start + i], dtype));
    if (isnan(ax)) return NAN;
    if (ax > a) a = ax;
  }
  return a;
}

/* Codes of one block given its absmax a.  Returns the codes in out[0..len). */
static void or_block_codes(const uint16_t* w, int dtype, int64_t start, int len, float a,
                           const float mids[15], int* out) {
  if (a == 0.0f) { /* all-zero block: the exact zero level */
    for (int i = 0; i < len; ++i) out[i] = 7;
    return;
  }
  float scale = 1.0f;
  float as = a;
  if (a < 0x1p-126f) { /* absmax below the normal range: scale the block by 2^64 first */
    scale = 0x1p64f;
    as = a * scale;
  }
  float r = 1.0f / as; /* one correctly rounded reciprocal per block */
  for (int i = 0; i < len; ++i) {
    float x = or_load(w[start + i], dtype) * scale;
    float v = x * r;
    out[i] = or_code_of(v, mids);
  }
}

static int or_is_finite_block(const uint16_t* w, int dtype, int64_t start, int len) {
  for (int i = 0; i < len; ++i)
    if (!isfinite(or_load(w[start + i], dtype))) return 0;
  return 1;
}

/* Blockwise absmax NF4 quantization with nibble packing.
   packed: ceil(n/2) bytes (may be NULL); absmax: ceil(n/64) floats (may be NULL).
   *nonfinite is set to 1 if any element is NaN or infinite (left untouched otherwise). */
void oracle_quantize(const uint16_t* w, int dtype, int64_t n, const float levels[16],
                     const float mids[15], uint8_t* packed, float* absmax, int* nonfinite) {
  (void)levels;
  int codes[OR_BLOCK];
  int64_t nb = (n + OR_BLOCK - 1) / OR_BLOCK;
  if (packed) memset(packed, 0, (size_t)((n + 1) / 2));
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * OR_BLOCK;
    int len = (int)(n - start < OR_BLOCK ? n - start : OR_BLOCK);
    float a = or_block_absmax(w, dtype, start, len);
    if (nonfinite && !or_is_finite_block(w, dtype, start, len)) *nonfinite = 1;
    or_block_codes(w, dtype, start, len, a, mids, codes);
    if (absmax) absmax[b] = a;
    if (packed)
      for (int i = 0; i < len; ++i) {
        int64_t e = start + i;
        if ((e & 1) == 0)
          packed[e >> 1] |= (uint8_t)(codes[i] << 4);
        else
          packed[e >> 1] |= (uint8_t)codes[i];
      }
  }
}

/* ------------------------------------------------------------ layer error */

/* Relative Frobenius NF4 reconstruction error of one layer ([AQLoRA/abs]).
   sq_err = sum (x - w_hat)^2, sq_w = sum x^2 (binary64, element order),
   rel = sqrt(sq_err / sq_w) (0 when sq_w == 0). */
void oracle_layer_error(const uint16_t* w, int dtype, int64_t n, const float levels[16],
                        const float mids[15], double* sq_err, double* sq_w, float* rel) {
  int codes[OR_BLOCK];
  double se = 0.0, sw = 0.0;
  int64_t nb = (n + OR_BLOCK - 1) / OR_BLOCK;
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * OR_BLOCK;
    int len = (int)(n - start < OR_BLOCK ? n - start : OR_BLOCK);
    float a = or_block_absmax(w, dtype, start, len);
    or_block_codes(w, dtype, start, len, a, mids, codes);
    for (int i = 0; i < len; ++i) {
      float x = or_load(w[start + i], dtype);
      float prod = levels[codes[i]] * a;
      float what = or_load(or_round_to_dtype(prod, dtype), dtype);
      double d = (double)x - (double)what;
      se += d * d;
      sw += (double)x * (double)x;
    }
  }
  *sq_err = se;
  *sq_w = sw;
  double e = sw == 0.0 ? 0.0 : sqrt(se / sw);
  if (isnan(se) || isnan(sw)) e = NAN;
  *rel = (float)e;
}

/* ------------------------------------------------------ double quantization */

/* Double quantization of one layer's absmax array ([QLoRA/HIW], [QLE/DQ]).
   codes8: nb bytes; scales: ceil(nb/256) floats.  A block of constants whose maximum is
   NaN or infinite gets codes 0, stores that maximum as its scale and sets *nonfinite. */
void oracle_double_quant(const float* absmax, int64_t nb, uint8_t* codes8, float* scales,
                         int* nonfinite) {
  int64_t nd = (nb + OR_DQ_BLOCK - 1) / OR_DQ_BLOCK;
  for (int64_t d = 0; d < nd; ++d) {
    int64_t start = d * OR_DQ_BLOCK;
    int64_t len = nb - start < OR_DQ_BLOCK ? nb - start : OR_DQ_BLOCK;
    float s = 0.0f;
    int bad = 0;
    for (int64_t i = 0; i < len; ++i) {
      float a = absmax[start + i];
      if (isnan(a)) bad = 1;
      if (a > s) s = a;
    }
    if (bad) s = NAN;
    scales[d] = s;
    if (!isfinite(s)) {
      if (nonfinite) *nonfinite = 1;
      for (int64_t i = 0; i < len; ++i) codes8[start + i] = 0;
      continue;
    }
    for (int64_t i = 0; i < len; ++i) {
      if (s == 0.0f) {
        codes8[start + i] = 0;
        continue;
      }
      float t = absmax[start + i] / s; /* correctly rounded divide */
      float u = t * 255.0f;
      float c = nearbyintf(u); /* ties to even */
      codes8[start + i] = (uint8_t)c;
    }
  }
}

/* ------------------------------------------------ mean-centred double quantization */

/* A second, optional DQ format ([QLoRA/HIW] gives only the 0.37-bit saving; centring the
   constants on their mean before a symmetric 8-bit code is a reading from outside the
   pages).  Per block of 256 constants (the last block may hold only len of them):
   (1) S = their sum in binary64 over a balanced binary tree of the 256 slots in index
       order (slot i + 1 pairs with slot i first, then pairs of pairs ...; the missing
       slots of a short block hold +0);
   (2) mean mu = fl32(fl64(S / len));
   (3) c_i = fl(a_i - mu); h = max |c_i|;
   (4) q_i = rint_even(fl(fl(c_i / h) * 127)) in [-127, 127], stored code8 = q_i + 128
       (h = 0: every code 128);
   (5) the constant a dequantization rebuilds: a'_i = fl(fl(fl(q_i / 127) * h) + mu).
   Storage per block: 256 codes, h and mu: 8/64 + 64/(64*256) = 0.12890625 bits per weight,
   0.37109375 less than binary32 constants.  A NaN or infinite constant makes the block's
   mu or h non-finite: its codes are 0, h and mu are stored as computed, *nonfinite set. */
static double or_tree_sum(const double* v, int n) { /* n a power of two */
  if (n == 1) return v[0];
  return or_tree_sum(v, n / 2) + or_tree_sum(v + n / 2, n / 2);
}

void oracle_double_quant_centered(const float* absmax, int64_t nb, uint8_t* codes8,
                                  float* scales, float* means, int* nonfinite) {
  int64_t nd = (nb + OR_DQ_BLOCK - 1) / OR_DQ_BLOCK;
  double slot[OR_DQ_BLOCK];
  for (int64_t d = 0; d < nd; ++d) {
    int64_t start = d * OR_DQ_BLOCK;
    int64_t len = nb - start < OR_DQ_BLOCK ? nb - start : OR_DQ_BLOCK;
    for (int64_t i = 0; i < OR_DQ_BLOCK; ++i) slot[i] = i < len ? (double)absmax[start + i] : 0.0;
    double S = or_tree_sum(slot, OR_DQ_BLOCK);
    float mu = (float)(S / (double)len);
    float h = 0.0f;
    for (int64_t i = 0; i < len; ++i) {
      float c = fabsf(absmax[start + i] - mu);
      if (isnan(c) || c > h) h = c;
    }
    scales[d] = h;
    means[d] = mu;
    if (!isfinite(mu) || !isfinite(h)) {
      if (nonfinite) *nonfinite = 1;
      for (int64_t i = 0; i < len; ++i) codes8[start + i] = 0;
      continue;
    }
    for (int64_t i = 0; i < len; ++i) {
      if (h == 0.0f) {
        codes8[start + i] = 128;
        continue;
      }
      float c = absmax[start + i] - mu;
      float t = c / h; /* correctly rounded divide */
      float q = nearbyintf(t * 127.0f);
      codes8[start + i] = (uint8_t)(int)(q + 128.0f);
    }
  }
}

/* The constant block b rebuilds from mean-centred DQ storage (step 5 above). */
static float or_centered_constant(const uint8_t* codes8, const float* scales,
                                  const float* means, int64_t b) {
  float t = (float)((int)codes8[b] - 128) / 127.0f;
  float u = t * scales[b / OR_DQ_BLOCK];
  return u + means[b / OR_DQ_BLOCK];
}

/* NF4 -> 16-bit from mean-centred DQ storage: as oracle_dequantize with the constant of
   or_centered_constant. */
void oracle_dequantize_centered(const uint8_t* packed, const uint8_t* codes8,
                                const float* scales, const float* means, int64_t n,
                                int out_dtype, const float levels[16], uint16_t* out) {
  for (int64_t e = 0; e < n; ++e) {
    float a = or_centered_constant(codes8, scales, means, e / OR_BLOCK);
    uint8_t byte = packed[e >> 1];
    int code = (e & 1) == 0 ? (byte >> 4) : (byte & 15);
    out[e] = or_round_to_dtype(levels[code] * a, out_dtype);
  }
}

/* The layer error of a model stored in NF4 with mean-centred DQ: as oracle_layer_error_dq
   with the constant of or_centered_constant.  Returns 0, or -1 if memory runs out. */
int oracle_layer_error_dqc(const uint16_t* w, int dtype, int64_t n, const float levels[16],
                           const float mids[15], double* sq_err, double* sq_w, float* rel) {
  int64_t nb = (n + OR_BLOCK - 1) / OR_BLOCK;
  int64_t nd = (nb + OR_DQ_BLOCK - 1) / OR_DQ_BLOCK;
  float* absmax = (float*)calloc((size_t)nb, sizeof(float));
  uint8_t* codes8 = (uint8_t*)calloc((size_t)nb, 1);
  float* scales = (float*)calloc((size_t)nd, sizeof(float));
  float* means = (float*)calloc((size_t)nd, sizeof(float));
  if (!absmax || !codes8 || !scales || !means) {
    free(absmax);
    free(codes8);
    free(scales);
    free(means);
    return -1;
  }
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * OR_BLOCK;
    int len = (int)(n - start < OR_BLOCK ? n - start : OR_BLOCK);
    absmax[b] = or_block_absmax(w, dtype, start, len);
  }
  oracle_double_quant_centered(absmax, nb, codes8, scales, means, NULL);
  int codes[OR_BLOCK];
  double se = 0.0, sw = 0.0;
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * OR_BLOCK;
    int len = (int)(n - start < OR_BLOCK ? n - start : OR_BLOCK);
    float a_dq = or_centered_constant(codes8, scales, means, b);
    or_block_codes(w, dtype, start, len, absmax[b], mids, codes);
    for (int i = 0; i < len; ++i) {
      float x = or_load(w[start + i], dtype);
      float what = or_load(or_round_to_dtype(levels[codes[i]] * a_dq, dtype), dtype);
      double d = (double)x - (double)what;
      se += d * d;
      sw += (double)x * (double)x;
    }
  }
  free(absmax);
  free(codes8);
  free(scales);
  free(means);
  *sq_err = se;
  *sq_w = sw;
  double e = sw == 0.0 ? 0.0 : sqrt(se / sw);
  if (isnan(se) || isnan(sw)) e = NAN;
  *rel = (float)e;
  return 0;
}

/* ------------------------------------------------ DQ-absmax layer error */

/* The layer error of a stored NF4 + DQ model ([QLoRA/HIW]: the constants are quantized in
   turn and the weights are dequantized from them).  In order: (1) the binary32 absmax of
   every block; (2) double quantization of those constants (oracle_double_quant); (3) each
   block's reconstruction constant a' = fl(fl(code8/255) * s); (4) codes from the binary32
   absmax, as in oracle_quantize; (5) w_hat = dtype_rn(fl(q[code] * a')) and the sums of
   oracle_layer_error.  Returns 0, or -1 if memory runs out. */
int oracle_layer_error_dq(const uint16_t* w, int dtype, int64_t n, const float levels[16],
                          const float mids[15], double* sq_err, double* sq_w, float* rel) {
  int64_t nb = (n + OR_BLOCK - 1) / OR_BLOCK;
  int64_t nd = (nb + OR_DQ_BLOCK - 1) / OR_DQ_BLOCK;
  float* absmax = (float*)calloc((size_t)nb, sizeof(float));
  uint8_t* codes8 = (uint8_t*)calloc((size_t)nb, 1);
  float* scales = (float*)calloc((size_t)nd, sizeof(float));
  if (!absmax || !codes8 || !scales) {
    free(absmax);
    free(codes8);
    free(scales);
    return -1;
  }
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * OR_BLOCK;
    int len = (int)(n - start < OR_BLOCK ? n - start : OR_BLOCK);
    absmax[b] = or_block_absmax(w, dtype, start, len);
  }
  oracle_double_quant(absmax, nb, codes8, scales, NULL);
  int codes[OR_BLOCK];
  double se = 0.0, sw = 0.0;
  for (int64_t b = 0; b < nb; ++b) {
    int64_t start = b * OR_BLOCK;
    int len = (int)(n - start < OR_BLOCK ? n - start : OR_BLOCK);
    float frac = (float)codes8[b] / 255.0f;
    float a_dq = frac * scales[b / OR_DQ_BLOCK];
    or_block_codes(w, dtype, start, len, absmax[b], mids, codes);
    for (int i = 0; i < len; ++i) {
      float x = or_load(w[start + i], dtype);
      float prod = levels[codes[i]] * a_dq;
      float what = or_load(or_round_to_dtype(prod, dtype), dtype);
      double d = (double)x - (double)what;
      se += d * d;
      sw += (double)x * (double)x;
    }
  }
  free(absmax);
  free(codes8);
  free(scales);
  *sq_err = se;
  *sq_w = sw;
  double e = sw == 0.0 ? 0.0 : sqrt(se / sw);
  if (isnan(se) || isnan(sw)) e = NAN;
  *rel = (float)e;
  return 0;
}

/* ------------------------------------------------------------- dequantize */

/* NF4 -> 16-bit ([QLoRA/HIW]: the 16-bit values a training pass computes with).
   With codes8 != NULL the block constant is a' = fl(fl(code8/255) * scale[b/256]);
   otherwise a' = absmax[b].  out: n 16-bit values of out_dtype. */
void oracle_dequantize(const uint8_t* packed, const uint8_t* codes8, const float* scales,
                       const float* absmax, int64_t n, int out_dtype, const float levels[16],
                       uint16_t* out) {
  for (int64_t e = 0; e < n; ++e) {
    int64_t b = e / OR_BLOCK;
    float a;
    if (codes8) {
      float frac = (float)codes8[b] / 255.0f;
      a = frac * scales[b / OR_DQ_BLOCK];
    } else {
      a = absmax[b];
    }
    uint8_t byte = packed[e >> 1];
    int code = (e & 1) == 0 ? (byte >> 4) : (byte & 15);
    float prod = levels[code] * a;
    out[e] = or_round_to_dtype(prod, out_dtype);
  }
}

/* ------------------------------------------------ linear layer on NF4 weights */

/* The forward product of a layer kept in NF4 + DQ ([QLoRA/HIW]: a training pass computes
   with 16-bit values rebuilt from the 4-bit storage): y = x w_hat^T with
   x: M x K 16-bit (x_dtype), row-major; w_hat: the N x K layer rebuilt in w_dtype from its
   packed codes, codes8 and scales exactly as oracle_dequantize does; y: M x N in binary64
   (every product and sum exact up to binary64 rounding).  yabs (optional) receives
   sum_k |x_mk| |w_hat_nk|, the scale of the rounding error a binary32 accumulation may
   make.  Returns 0, or -1 if memory runs out. */
int oracle_nf4_linear(const uint16_t* x, int x_dtype, int64_t M, int64_t K,
                      const uint8_t* packed, const uint8_t* codes8, const float* scales,
                      int64_t N, int w_dtype, const float levels[16], double* y,
                      double* yabs) {
  uint16_t* row16 = (uint16_t*)calloc((size_t)K, sizeof(uint16_t));
  double* wrow = (double*)calloc((size_t)K, sizeof(double));
  double* xv = (double*)calloc((size_t)(M * K), sizeof(double));
  if (!row16 || !wrow || !xv) {
    free(row16);
    free(wrow);
    free(xv);
    return -1;
  }
  for (int64_t i = 0; i < M * K; ++i) xv[i] = (double)or_load(x[i], x_dtype);
  for (int64_t n = 0; n < N; ++n) {
    /* row n of w_hat: elements n*K .. n*K + K - 1 of the flattened layer */
    for (int64_t k = 0; k < K; ++k) {
      int64_t e = n * K + k;
      int64_t b = e / OR_BLOCK;
      float frac = (float)codes8[b] / 255.0f;
      float a = frac * scales[b / OR_DQ_BLOCK];
      uint8_t byte = packed[e >> 1];
      int code = (e & 1) == 0 ? (byte >> 4) : (byte & 15);
      float prod = levels[code] * a;
      row16[k] = or_round_to_dtype(prod, w_dtype);
      wrow[k] = (double)or_load(row16[k], w_dtype);
    }
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        acc += xv[m * K + k] * wrow[k];
        aacc += fabs(xv[m * K + k] * wrow[k]);
      }
      y[m * N + n] = acc;
      if (yabs) yabs[m * N + n] = aacc;
    }
  }
  free(row16);
  free(wrow);
  free(xv);
  return 0;
}

/* ---------------------------------------------------------------- selection */

/* Incremental bytes of keeping an n-element layer in 16 bits instead of NF4 storage
   (packed nibbles + 8-bit DQ codes + fp32 DQ scales) ([AQLoRA/abs] 0.2 GiB reading). */
int64_t oracle_cost_bytes(int64_t n) {
  int64_t nb = (n + OR_BLOCK - 1) / OR_BLOCK;
  int64_t nd = (nb + OR_DQ_BLOCK - 1) / OR_DQ_BLOCK;
  return 2 * n - ((n + 1) / 2 + nb + 4 * nd);
}

/* does layer j rank before layer i?  (score desc, NaN last, index asc) */
static int or_before(const float* e, int j, int i) {
  int nj = isnan(e[j]), ni = isnan(e[i]);
  if (nj != ni) return ni; /* the non-NaN one first */
  if (!nj && e[j] != e[i]) return e[j] > e[i];
  return j < i;
}

/* Top-K under a byte budget ([AQLoRA/abs], [AQLoRA/TD]).  k_cap < 0 means no cap.
   sel receives the kept layer indices in rank order; returns -1 on bad arguments. */
int oracle_select_topk(const float* e, const int64_t* cost, int L, int64_t budget, int k_cap,
                       int* sel, int* k_out) {
  if (L < 0 || budget < 0) return -1;
  int order[L > 0 ? L : 1];
  for (int i = 0; i < L; ++i) order[i] = i;
  /* selection sort by the rank relation: O(L^2), plain */
  for (int a = 0; a < L; ++a) {
    int best = a;
    for (int b = a + 1; b < L; ++b)
      if (or_before(e, order[b], order[best])) best = b;
    int t = order[a];
    order[a] = order[best];
    order[best] = t;
  }
  int64_t used = 0;
  int k = 0;
  for (int r = 0; r < L; ++r) {
    if (k_cap >= 0 && k >= k_cap) break;
    int l = order[r];
    if (used + cost[l] > budget) break; /* stop at the first layer that does not fit */
    used += cost[l];
    sel[k++] = l;
  }
  *k_out = k;
  return 0;
}

/* Block-level selection for the speed setting ([AQLoRA/abs]: a speed setting adapts only
   the top blocks, so the backward pass stops early; [AQLoRA/TD]: it promotes only the top
   blocks).  Each layer l belongs to transformer block block_of[l] in [0, B).  A block costs
   the sum of its layers' costs.  Its score is the relative error of all its layers together,
   sqrt(sum sq_err / sum sq_w) with the sums in binary64 in layer order (0 when the block's
   sum sq_w is 0).  order 0 ranks the blocks by depth, last block first: the plain reading
   of "top blocks".  order 1 ranks them by score (desc, NaN last, index asc).  The kept
   blocks are the longest prefix of the ranking whose total cost fits the budget.  rank[B]
   receives the whole ranking, block_err[B] the scores and *k_out the number kept.
   Returns 0, or -1 for invalid arguments. */
int oracle_select_blocks(const double* sq_err, const double* sq_w, const int* block_of,
                         const int64_t* cost, int L, int B, int64_t budget, int order,
                         int* rank, float* block_err, int* k_out) {
  if (L < 0 || B < 1 || budget < 0 || (order != 0 && order != 1)) return -1;
  for (int l = 0; l < L; ++l)
    if (block_of[l] < 0 || block_of[l] >= B) return -1;
  int64_t bcost[B];
  for (int b = 0; b < B; ++b) {
    double se = 0.0, sw = 0.0;
    bcost[b] = 0;
    for (int l = 0; l < L; ++l) {
      if (block_of[l] != b) continue;
      se += sq_err[l];
      sw += sq_w[l];
      bcost[b] += cost[l];
    }
    double e = sw == 0.0 ? 0.0 : sqrt(se / sw);
    if (isnan(se) || isnan(sw)) e = NAN;
    block_err[b] = (float)e;
  }
  for (int i = 0; i < B; ++i) rank[i] = order == 0 ? B - 1 - i : i;
  if (order == 1) {
    for (int a = 0; a < B; ++a) {
      int best = a;
      for (int c = a + 1; c < B; ++c)
        if (or_before(block_err, rank[c], rank[best])) best = c;
      int t = rank[a];
      rank[a] = rank[best];
      rank[best] = t;
    }
  }
  int64_t used = 0;
  int k = 0;
  while (k < B && used + bcost[rank[k]] <= budget) used += bcost[rank[k++]];
  *k_out = k;
  return 0;
}

/* bit helpers exported for the tests' conversion pins */
uint16_t oracle_f32_to_dtype_bits(float f, int dtype) { return or_round_to_dtype(f, dtype); }
float oracle_dtype_bits_to_f32(uint16_t h, int dtype) { return or_load(h, dtype); }
uint32_t oracle_f32_bits(float f) { return or_f32_to_bits(f); }
