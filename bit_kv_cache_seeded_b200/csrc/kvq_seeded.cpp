// The method's seeded random draws on the host: the +-1 diagonal of the randomized Hadamard
// rotation and the Gaussian QJL sketch matrix ("TurboQuant vs OSCAR vs EpiCache", section
// "Quantization frontiers: TurboQuant and OSCAR": a data-oblivious random rotation, then a 1-bit
// Johnson-Lindenstrauss sketch of the residual). The generator is the counter-based splitmix64
// stream and Box-Muller transform that kvq.h defines next to kvq_draw_rotation_signs; a cache
// given no arrays draws its tables here, so a C caller reproduces a seeded cache from two seeds.
#include <cmath>
#include <cstdint>

#include "kvq.h"

namespace {

constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

uint64_t draw(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1) * kGolden;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

double uniform53(uint64_t seed, uint64_t i) { return (double)(draw(seed, i) >> 11) * 0x1.0p-53; }

}  // namespace

extern "C" kvq_status kvq_draw_rotation_signs(uint64_t seed, int32_t n, int8_t* out) {
  if (!out || n <= 0) return KVQ_ERR_INVALID_ARG;
  for (int32_t i = 0; i < n; ++i) out[i] = (draw(seed, (uint64_t)i) & 1u) ? int8_t(-1) : int8_t(1);
  return KVQ_OK;
}

extern "C" kvq_status kvq_draw_qjl_matrix(uint64_t seed, int32_t m, int32_t d, float* out) {
  if (!out || m <= 0 || d <= 0) return KVQ_ERR_INVALID_ARG;
  const double two_pi = 2.0 * 3.141592653589793;
  const uint64_t n = (uint64_t)m * (uint64_t)d;
  for (uint64_t k = 0; k < n; ++k) {
    const double u1 = uniform53(seed, 2 * k), u2 = uniform53(seed, 2 * k + 1);
    const double g = std::sqrt(-2.0 * std::log1p(-u1)) * std::cos(two_pi * u2);
    out[k] = (float)g;
  }
  return KVQ_OK;
}
