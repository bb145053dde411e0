#include "nf4_host.h"

#include <cmath>
#include <mutex>

namespace qlora {

namespace {

double normal_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }

// Phi^{-1}(p) for 0.5 <= p < 1 by Newton's method from 0 (Phi is concave on
// x >= 0, so the iterates increase monotonically to the root).
double normal_quantile_upper(double p) {
  const double inv_sqrt_2pi = 0.39894228040143267794;
  double x = 0.0;
  for (int it = 0; it < 200; ++it) {
    const double f = normal_cdf(x) - p;
    const double step = f / (inv_sqrt_2pi * std::exp(-0.5 * x * x));
    const double nx = x - step;
    if (nx == x) break;
    x = nx;
  }
  return x;
}

// Levels plus the encoder's boundaries for a sorted table of 16 levels.
Nf4Params with_boundaries(const float q[16]) {
  Nf4Params P{};
  for (int i = 0; i < 16; ++i) P.q[i] = q[i];
  for (int j = 0; j < 15; ++j) {
    const double mid = 0.5 * (static_cast<double>(P.q[j]) + static_cast<double>(P.q[j + 1]));  // exact
    float u = static_cast<float>(mid);
    if (static_cast<double>(u) <= mid) u = std::nextafter(u, INFINITY);  // smallest float > mid
    const float below = std::nextafter(u, -INFINITY);
    P.bnd[j] = 0.5 * (static_cast<double>(below) + static_cast<double>(u));  // exact (25 bits)
  }
  return P;
}

Nf4Params build_nf4() {
  float q[16];
  nf4_levels(q);
  return with_boundaries(q);
}

// FP4: the float with 1 sign, 2 exponent and 1 mantissa bit; its seven
// non-zero magnitudes 0.5, 1, 1.5, 2, 3, 4, 6 divided by the largest.  Int4:
// k / 7.  Sorted with the zero at index 7; index 15 repeats +1, so that the
// nearest-level rule (ties to the lower index) never picks it.
Nf4Params build_fp4() {
  const double mags[7] = {0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  float q[16];
  for (int i = 0; i < 7; ++i) {
    q[6 - i] = static_cast<float>(-mags[i] / 6.0);
    q[8 + i] = static_cast<float>(mags[i] / 6.0);
  }
  q[7] = 0.0f;
  q[15] = q[14];
  return with_boundaries(q);
}

Nf4Params build_int4() {
  float q[16];
  for (int k = -7; k <= 7; ++k) q[k + 7] = static_cast<float>(k / 7.0);
  q[15] = q[14];
  return with_boundaries(q);
}

}  // namespace

void nf4_levels(float out[16]) {
  const double delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  double v[16];
  int n = 0;
  // negative side: 7 probabilities from delta towards 0.5 (0.5 itself excluded)
  const double step7 = (0.5 - delta) / 7.0;
  for (int i = 0; i < 7; ++i) v[n++] = -normal_quantile_upper(delta + i * step7);
  v[n++] = 0.0;
  const double step8 = (0.5 - delta) / 8.0;
  for (int i = 7; i >= 0; --i) v[n++] = normal_quantile_upper(delta + i * step8);
  const double top = v[15];
  for (int i = 0; i < 16; ++i) out[i] = static_cast<float>(v[i] / top);
}

const Nf4Params& nf4_params() { return code_params(0); }

const Nf4Params* code_params_or_null(int code) {
  static std::once_flag once;
  static Nf4Params P[3];
  std::call_once(once, [] {
    P[0] = build_nf4();
    P[1] = build_fp4();
    P[2] = build_int4();
  });
  return (code >= 0 && code < 3) ? &P[code] : nullptr;
}

const Nf4Params& code_params(int code) { return *code_params_or_null(code >= 0 && code < 3 ? code : 0); }

}  // namespace qlora
