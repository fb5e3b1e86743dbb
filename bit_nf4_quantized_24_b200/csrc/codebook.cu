// The NF4 codebook of this library, computed on the host at first use.
//
// katajob, "NF4: 4-bit NormalFloat": 16 levels placed for values drawn from a
// zero-centred normal.  Construction used here: equal-probability quantiles
// of N(0, 1) on each side of an exact zero -- 8 positive levels at
// p_j = 1/2 + j (delta - 1/2) / 8 and 7 negative levels at the mirror of
// q_j = 1/2 + j (delta - 1/2) / 7 -- all divided by the quantile of delta so
// the outermost levels are exactly -1 and +1.  delta = 1 - (1/32 + 1/30) / 2
// centres the outermost probability between the top bins of a 16-way and a
// 15-way equal-mass split.
//
// The quantile is found by Newton's method on Phi(x) - p, Phi(x) =
// erfc(-x / sqrt 2) / 2, started from the rational approximation of
// Abramowitz & Stegun 26.2.23.  Levels are rounded once to fp32; decision
// midpoints are fl32(L_i + L_{i+1}) * 0.5 in fp32.
#include <cmath>
#include <mutex>

#include "internal.h"

namespace qn {

namespace {

double phi(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }
double phi_density(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * 3.14159265358979323846); }

// Standard normal quantile for p in (1/2, 1).
double upper_quantile(double p) {
  const double q = 1.0 - p;
  const double t = std::sqrt(-2.0 * std::log(q));
  double x = t - (2.515517 + 0.802853 * t + 0.010328 * t * t) /
                     (1.0 + 1.432788 * t + 0.189269 * t * t + 0.001308 * t * t * t);
  for (int i = 0; i < 100; ++i) {
    const double step = (phi(x) - p) / phi_density(x);
    x -= step;
    if (std::fabs(step) <= 1e-17 * std::fabs(x)) break;
  }
  return x;
}

HostCodebook build() {
  const double delta = 1.0 - (1.0 / 32.0 + 1.0 / 30.0) / 2.0;
  const double z = upper_quantile(delta);
  double lv[16];
  lv[7] = 0.0;
  for (int j = 1; j <= 8; ++j) lv[7 + j] = upper_quantile(0.5 + (delta - 0.5) * j / 8.0) / z;
  for (int j = 1; j <= 7; ++j) lv[7 - j] = -upper_quantile(0.5 + (delta - 0.5) * j / 7.0) / z;
  HostCodebook cb;
  for (int i = 0; i < 16; ++i) cb.levels.v[i] = static_cast<float>(lv[i]);
  for (int i = 0; i < 15; ++i) {
    const float s = cb.levels.v[i] + cb.levels.v[i + 1];
    cb.mids.v[i] = s * 0.5f;
  }
  return cb;
}

}  // namespace

const HostCodebook& host_codebook() {
  static HostCodebook cb;
  static std::once_flag once;
  std::call_once(once, [] { cb = build(); });
  return cb;
}

}  // namespace qn
