// The 16 NF4 (4-bit NormalFloat) levels, derived on the host at first use.
//
// The pages (solutions index, grouped-nf4-gemm table; "experts4bit-qlora"
// limits list) name the bitsandbytes NF4 format but print no levels.  The
// levels here follow the NormalFloat construction of the QLoRA paper
// (Dettmers et al., 2023, "4-bit NormalFloat Quantization"): standard-normal
// quantiles at 9 evenly spaced probabilities from delta down to 1/2 for the
// positive side and at 8 for the negative side, the shared zero kept once,
// all divided by the largest quantile so the levels span [-1, 1].  The end
// probability is delta = 1 - (1/30 + 1/32) / 2.
//
// The inverse normal CDF is solved here by safeguarded Newton iteration on
// Phi(z) = 0.5 * erfc(-z / sqrt 2) in double precision; the levels are then
// rounded once to fp32, and each decision midpoint is the fp32 rounding of
// the exact mean of two neighbouring fp32 levels.
#include <cmath>
#include <mutex>

#include "e4b_internal.h"

namespace e4b {
namespace {

double normal_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }

// z with Phi(z) = p, for 0.5 <= p < 1.
double normal_quantile_upper(double p) {
  if (p == 0.5) return 0.0;
  double lo = 0.0, hi = 40.0, z = 1.0;
  for (int it = 0; it < 100; ++it) {
    const double f = normal_cdf(z) - p;
    if (f < 0.0) lo = z; else hi = z;
    const double dens = std::exp(-0.5 * z * z) / std::sqrt(2.0 * M_PI);
    double zn = z - f / dens;
    if (!(zn > lo && zn < hi)) zn = 0.5 * (lo + hi);
    if (zn == z) break;   // converged (or oscillating at the last bit: ends at the cap)
    z = zn;
  }
  return z;
}

Nf4Table build_table() {
  const double delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  double pos[8], neg[7];
  for (int i = 0; i < 8; ++i) pos[i] = normal_quantile_upper(delta + i * (0.5 - delta) / 8.0);
  for (int i = 0; i < 7; ++i) neg[i] = normal_quantile_upper(delta + i * (0.5 - delta) / 7.0);
  const double top = pos[0];
  double lv[16];
  for (int i = 0; i < 7; ++i) lv[i] = -neg[i] / top;          // ascending: -1 ... smallest negative
  lv[7] = 0.0;
  for (int i = 0; i < 8; ++i) lv[8 + i] = pos[7 - i] / top;    // smallest positive ... 1
  Nf4Table t;
  for (int i = 0; i < 16; ++i) t.level[i] = static_cast<float>(lv[i]);
  for (int i = 0; i < 15; ++i)
    t.mid[i] = static_cast<float>((static_cast<double>(t.level[i]) + static_cast<double>(t.level[i + 1])) / 2.0);
  return t;
}

}  // namespace

const Nf4Table& nf4_table() {
  static Nf4Table table;
  static std::once_flag once;
  std::call_once(once, [] { table = build_table(); });
  return table;
}

}  // namespace e4b
