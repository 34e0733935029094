// codebook.cpp -- host side of libaqnf4: the NF4 codebook, the kernels' lookup tables,
// status strings, the cost model and the launch counter.
//
// NF4 ("QLoRA", "How It Works"; "QLoRA Explained", "NF4"): 16 levels placed so that
// normally distributed weights fall evenly on them.  Here, as in the quantile construction
// the pages describe, the positive levels are standard-normal quantiles at probabilities
// spaced evenly from 1/2 (left out, it would give 0) up to p_max, likewise the negative
// ones, plus an exact 0, all scaled so the outermost level is 1.

#include <atomic>
#include <cmath>
#include <limits>
#include <mutex>

#include "internal.h"

namespace aqnf4 {
namespace {

double std_normal_cdf(double z) { return 0.5 * std::erfc(-z * 0.70710678118654752440); }

double std_normal_pdf(double z) { return 0.39894228040143267794 * std::exp(-0.5 * z * z); }

// Standard-normal quantile for p in [1/2, 1) by Newton's method on the CDF.  The CDF is
// concave on z >= 0, so Newton iterates started at 0 increase monotonically to the root;
// iterate until the step no longer changes z.
double std_normal_quantile_upper(double p) {
  double z = 0.0;
  for (int it = 0; it < 200; ++it) {
    double step = (std_normal_cdf(z) - p) / std_normal_pdf(z);
    double next = z - step;
    if (next == z) break;
    z = next;
  }
  return z;
}

std::atomic<uint64_t> g_launches{0};

Tables g_tables;
const Tables* g_tables_ptr = nullptr;
std::once_flag g_tables_once;

// Slot curve k(v) = round(a v + b v^3 + 8) for the default codebook: the max-margin odd
// cubic (both coefficients exact in binary32).  check_slot_curve proves it below.
constexpr float kCurveA = 11.71875f;
constexpr float kCurveB = -4.125f;

// h(v) = a v + b v^3 + 8.5; the kernel's round-to-nearest of a v + b v^3 + 8 is floor(h)
// away from ties, and either neighbour at a tie.  For v in (mid_{j-1}, mid_j] (with the
// ends -1 - 2^-20 and 1 + 2^-20 outside the first and last midpoints) the slot must be j or
// j + 1, i.e. j + margin <= h(v) <= j + 2 - margin.  A cubic's extremes on an interval are
// at its ends or its critical points, so checking those points in binary64 is a proof; the
// margin (1/64 of a slot) dwarfs the error of evaluating h in binary32 (below 1e-5).
bool check_slot_curve(const Tables& t) {
  const double a = t.curve_a, b = t.curve_b, margin = 1.0 / 64.0;
  auto h = [&](double v) { return a * v + b * v * v * v + 8.5; };
  const double ends = 1.0 + std::ldexp(1.0, -20);
  const double crit = (b < 0.0 && a > 0.0) ? std::sqrt(a / (-3.0 * b)) : -1.0;
  for (int j = 0; j < 16; ++j) {
    const double lo = j == 0 ? -ends : t.mid[j - 1];
    const double hi = j == 15 ? ends : t.mid[j];
    double hmin = std::fmin(h(lo), h(hi)), hmax = std::fmax(h(lo), h(hi));
    for (double c : {crit, -crit}) {
      if (crit > 0.0 && c > lo && c < hi) {
        hmin = std::fmin(hmin, h(c));
        hmax = std::fmax(hmax, h(c));
      }
    }
    if (hmin < j + margin || hmax > j + 2 - margin) return false;
  }
  return true;
}

bool build_tables(Tables& t) {
  if (aqnf4_codebook(0.0, t.level, t.mid) != AQNF4_OK) return false;
  t.curve_a = kCurveA;
  t.curve_b = kCurveB;
  if (!check_slot_curve(t)) return false;
  for (int k = 0; k < 32; ++k) {
    t.slot_mid[k] = k == 0    ? -std::numeric_limits<float>::infinity()
                    : k <= 15 ? t.mid[k - 1]
                              : std::numeric_limits<float>::infinity();
    t.slot_level[k] = k == 0 ? t.level[0] : k <= 16 ? t.level[k - 1] : t.level[15];
  }
  return true;
}

}  // namespace

const Tables* default_tables() {
  std::call_once(g_tables_once, [] {
    if (build_tables(g_tables)) g_tables_ptr = &g_tables;
  });
  return g_tables_ptr;
}

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int current_sm_count() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return sms;
}

}  // namespace aqnf4

extern "C" {

const char* aqnf4_status_string(aqnf4_status st) {
  switch (st) {
    case AQNF4_OK: return "ok";
    case AQNF4_ERR_INVALID_ARG: return "invalid argument";
    case AQNF4_ERR_ALIGNMENT: return "misaligned pointer";
    case AQNF4_ERR_DTYPE: return "unsupported dtype";
    case AQNF4_ERR_NONFINITE: return "non-finite input";
    case AQNF4_ERR_CUDA: return "CUDA error";
    case AQNF4_ERR_TIMEOUT: return "bounded wait timed out";
    case AQNF4_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
  }
  return "unknown status";
}

aqnf4_status aqnf4_codebook(double p_max, float levels[16], float mids[15]) {
  if (!levels || !mids) return AQNF4_ERR_INVALID_ARG;
  if (p_max <= 0.0) p_max = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
  if (!(p_max > 0.5 && p_max < 1.0)) return AQNF4_ERR_INVALID_ARG;
  double q[16];
  int n = 0;
  const double span = p_max - 0.5;
  for (int k = 0; k < 7; ++k) q[n++] = -aqnf4::std_normal_quantile_upper(p_max - k * span / 7.0);
  q[n++] = 0.0;
  for (int k = 0; k < 8; ++k) q[n++] = aqnf4::std_normal_quantile_upper(p_max - k * span / 8.0);
  // q[0..6] ascend (most negative first), q[7] = 0, q[8..15] descend: reorder ascending.
  double asc[16];
  for (int i = 0; i < 7; ++i) asc[i] = q[i];
  asc[7] = 0.0;
  for (int i = 0; i < 8; ++i) asc[8 + i] = q[15 - i];
  const double outer = asc[15];  // the quantile of p_max, the largest magnitude
  for (int i = 0; i < 16; ++i) levels[i] = static_cast<float>(asc[i] / outer);
  for (int j = 0; j < 15; ++j)
    mids[j] = static_cast<float>((static_cast<double>(levels[j]) + levels[j + 1]) * 0.5);
  return AQNF4_OK;
}

int64_t aqnf4_cost_bytes(int64_t n) {
  if (n < 1) return -1;
  const int64_t nb = (n + aqnf4::kBlock - 1) / aqnf4::kBlock;
  const int64_t nd = (nb + aqnf4::kDqBlock - 1) / aqnf4::kDqBlock;
  return 2 * n - ((n + 1) / 2 + nb + 4 * nd);
}

aqnf4_status aqnf4_slot_tables(float* curve, float* slot_mid, float* slot_level) {
  if (!curve || !slot_mid || !slot_level) return AQNF4_ERR_INVALID_ARG;
  const aqnf4::Tables* tb = aqnf4::default_tables();
  if (!tb) return AQNF4_ERR_CUDA;
  curve[0] = tb->curve_a;
  curve[1] = tb->curve_b;
  for (int k = 0; k < 32; ++k) {
    slot_mid[k] = tb->slot_mid[k];
    slot_level[k] = tb->slot_level[k];
  }
  return AQNF4_OK;
}

uint64_t aqnf4_launch_count(void) { return aqnf4::g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
