// Gaussian Lloyd-Max tables computed on the host at cache creation.
//
// "TurboQuant vs OSCAR vs EpiCache" (dothoosh.com), section "Quantization frontiers:
// TurboQuant and OSCAR": the rotated coordinates are close to N(0, 1), so one precomputed
// optimal scalar quantizer (Lloyd-Max) serves every coordinate. The table is the fixed point
// of the two optimality conditions, found in fp64 and rounded once to fp32:
//   centroid of a cell   = E[X | lo <= X < hi] = (pdf(lo) - pdf(hi)) / (cdf(hi) - cdf(lo))
//   boundary of two cells = midpoint of their centroids.
// N(0, 1) is even, so the table is odd; the two halves are averaged after every sweep so that
// the middle boundary is exactly 0.
#include <cmath>
#include <limits>

#include "kvq_internal.h"

namespace kvq {
namespace {

double normal_pdf(double x) {
  if (std::isinf(x)) return 0.0;
  return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI);
}

double normal_cdf(double x) {
  if (x == -std::numeric_limits<double>::infinity()) return 0.0;
  if (x == std::numeric_limits<double>::infinity()) return 1.0;
  return 0.5 * std::erfc(-x / std::sqrt(2.0));
}

}  // namespace

void lloyd_max_f32(int bits, float* centroids, float* thresholds) {
  const int L = 1 << bits;
  double c[8], nc[8], edge[9];
  for (int k = 0; k < L; ++k) c[k] = -2.0 + 4.0 * k / (L - 1);  // spread over [-2, 2]
  const double inf = std::numeric_limits<double>::infinity();
  for (int it = 0; it < 1000000; ++it) {
    edge[0] = -inf;
    edge[L] = inf;
    for (int k = 1; k < L; ++k) edge[k] = 0.5 * (c[k - 1] + c[k]);
    for (int k = 0; k < L; ++k)
      nc[k] = (normal_pdf(edge[k]) - normal_pdf(edge[k + 1])) /
              (normal_cdf(edge[k + 1]) - normal_cdf(edge[k]));
    double sym[8];
    for (int k = 0; k < L; ++k) sym[k] = 0.5 * (nc[k] - nc[L - 1 - k]);
    double delta = 0.0;
    for (int k = 0; k < L; ++k) {
      delta = std::fmax(delta, std::fabs(sym[k] - c[k]));
      c[k] = sym[k];
    }
    if (delta < 1e-15) break;
  }
  for (int k = 0; k < L; ++k) centroids[k] = static_cast<float>(c[k]);
  for (int k = 0; k + 1 < L; ++k) thresholds[k] = static_cast<float>(0.5 * (c[k] + c[k + 1]));
}

}  // namespace kvq
