// Host side of the codebook quantizer: the unit-sphere Lloyd-Max codebook.
//
// "orbitquant 0.2.0" (Features; Method Conformance): activations are
// quantized to the nearest centroid of one fixed codebook per (input
// dimension, bit width), an exact unit-sphere Lloyd-Max codebook.  A rotated,
// normalized activation row behaves as a uniform unit vector in R^d, whose
// coordinates have the density
//
//     f_d(t) = (1 - t^2)^((d - 3) / 2) / B(1/2, (d - 1) / 2),   -1 <= t <= 1.
//
// The codebook is the minimum mean-square-error quantizer of f_d with 2^bits
// levels, found by Lloyd's iteration: thresholds are the midpoints of adjacent
// centroids, and each centroid is the conditional mean of its cell,
//
//     c_i = M(t_(i-1), t_i) / (F(t_i) - F(t_(i-1))),
//     F(t) = 1/2 + sign(t) I_(t^2)(1/2, (d - 1)/2) / 2      (the CDF),
//     M(a, b) = ((1 - a^2)^((d-1)/2) - (1 - b^2)^((d-1)/2)) / ((d - 1) B(1/2, (d-1)/2)),
//
// I the regularized incomplete beta function, evaluated with its continued
// fraction (Abramowitz and Stegun 26.5.8, modified Lentz evaluation).
// Everything is double precision and runs on the host, once per (d, bits).
#include "hadq.h"

#include <cmath>
#include <vector>

namespace {

// Continued fraction of I_x(a, b) for x < (a + 1) / (a + b + 2).
double betacf(double a, double b, double x) {
  const double tiny = 1e-300, eps = 1e-16;
  double c = 1.0, d = 1.0 - (a + b) * x / (a + 1.0);
  if (std::fabs(d) < tiny) d = tiny;
  d = 1.0 / d;
  double h = d;
  for (int m = 1; m <= 10000; ++m) {
    const double m2 = 2.0 * m;
    double aa = m * (b - m) * x / ((a + m2 - 1.0) * (a + m2));   // even step
    d = 1.0 + aa * d;
    if (std::fabs(d) < tiny) d = tiny;
    c = 1.0 + aa / c;
    if (std::fabs(c) < tiny) c = tiny;
    d = 1.0 / d;
    h *= d * c;
    aa = -(a + m) * (a + b + m) * x / ((a + m2) * (a + m2 + 1.0));   // odd step
    d = 1.0 + aa * d;
    if (std::fabs(d) < tiny) d = tiny;
    c = 1.0 + aa / c;
    if (std::fabs(c) < tiny) c = tiny;
    d = 1.0 / d;
    const double del = d * c;
    h *= del;
    if (std::fabs(del - 1.0) < eps) break;
  }
  return h;
}

// Regularized incomplete beta I_x(a, b), 0 <= x <= 1.
double betai(double a, double b, double x) {
  if (x <= 0.0) return 0.0;
  if (x >= 1.0) return 1.0;
  const double lbt = std::lgamma(a + b) - std::lgamma(a) - std::lgamma(b) + a * std::log(x) + b * std::log1p(-x);
  if (x < (a + 1.0) / (a + b + 2.0)) return std::exp(lbt) * betacf(a, b, x) / a;
  return 1.0 - std::exp(lbt) * betacf(b, a, 1.0 - x) / b;
}

struct Marginal {
  double d, e, log_beta;   // e = (d - 1) / 2; log B(1/2, e)
  explicit Marginal(double dim) : d(dim), e((dim - 1.0) / 2.0) {
    log_beta = std::lgamma(0.5) + std::lgamma(e) - std::lgamma(0.5 + e);
  }
  double cdf(double t) const {
    if (t <= -1.0) return 0.0;
    if (t >= 1.0) return 1.0;
    const double half = 0.5 * betai(0.5, e, t * t);
    return t < 0 ? 0.5 - half : 0.5 + half;
  }
  double g(double t) const {   // (1 - t^2)^e
    const double w = 1.0 - t * t;
    return w <= 0.0 ? 0.0 : std::exp(e * std::log(w));
  }
  double first_moment(double a, double b) const {   // integral of t f_d(t) over [a, b]
    return (g(a) - g(b)) / ((d - 1.0) * std::exp(log_beta));
  }
  double quantile(double p) const {   // bisection on the CDF
    double lo = -1.0, hi = 1.0;
    for (int i = 0; i < 200 && hi - lo > 1e-17; ++i) {
      const double mid = 0.5 * (lo + hi);
      (cdf(mid) < p ? lo : hi) = mid;
    }
    return 0.5 * (lo + hi);
  }
};

}  // namespace

extern "C" {

hadq_status hadq_codebook(int64_t d, int bits, double* centroids, double* thresholds) {
  if (d < 2 || d > (int64_t(1) << 40) || bits < 1 || bits > 8 || centroids == nullptr || thresholds == nullptr)
    return HADQ_ERR_INVALID_ARG;
  const int levels = 1 << bits;
  const Marginal f(static_cast<double>(d));
  std::vector<double> c(levels), t(levels - 1);
  for (int i = 0; i < levels; ++i) c[i] = f.quantile((i + 0.5) / levels);
  for (int it = 0; it < 200000; ++it) {
    for (int i = 0; i + 1 < levels; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
    double moved = 0.0, cmax = 0.0;
    for (int i = 0; i < levels; ++i) {
      const double a = i == 0 ? -1.0 : t[i - 1], b = i == levels - 1 ? 1.0 : t[i];
      const double next = f.first_moment(a, b) / (f.cdf(b) - f.cdf(a));
      moved = std::fmax(moved, std::fabs(next - c[i]));
      c[i] = next;
      cmax = std::fmax(cmax, std::fabs(next));
    }
    if (moved <= 1e-13 * cmax) break;
  }
  for (int i = 0; i + 1 < levels; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
  for (int i = 0; i < levels; ++i) centroids[i] = c[i];
  for (int i = 0; i + 1 < levels; ++i) thresholds[i] = t[i];
  return HADQ_OK;
}

}  // extern "C"
