// Pieces shared by the two LM / LM_QJL / SIGN1 decode kernels (mma.sync in kvq_decode_mma.cu,
// tcgen05 in kvq_decode_tc.cu): constants of the integer formulation, the Walsh expansion of an
// odd Lloyd-Max table, and the compile-time layout of a cache tile.
//
// Walsh expansion ("TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant
// and OSCAR": a precomputed Lloyd-Max scalar quantizer per coordinate). The Lloyd-Max table of a
// symmetric density is odd, so with B_i = 2 b_i - 1 every code value is a signed sum of +-1 planes:
//   1 bit : c = a0 B0;   2 bits: c = a0 B0 + a1 B1
//   3 bits: c = a0 B0 + a1 B1 + a2 B2 + a3 B0B1B2,   B0B1B2 = 2 (b0 ^ b1 ^ b2) - 1
// and <q, c[code]> = sum_P 2 a_P <q, b_P> - (sum_P a_P) sum_j q_j over 0/1 "Walsh planes".
#pragma once

#include <cuda_bf16.h>

#include "kvq_internal.h"

namespace kvq {
namespace lmc {

constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)
constexpr float kSqrtHalfPi = 1.2533141373155003f;  // sqrt(pi/2)
constexpr int kQRange = 32639;                       // query term quantised to [-32639, 32639]
constexpr float kWRange = 8388608.f;                 // weights quantised below 2^23
constexpr float kRoundBias = 8388608.f;              // x + 2^23 (0 <= x < 2^23): bits = 0x4B000000 | rint(x)

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float load_q(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

template <int BITS> struct Walsh { static constexpr int P = BITS == 3 ? 4 : BITS; };

// 32-bit word of Walsh plane P from the stored bit-plane words (parity plane for 3 bits).
template <int BITS>
__device__ __forceinline__ uint32_t walsh_word(const uint32_t (&w)[3], int P) {
  if (BITS == 3 && P == 3) return w[0] ^ w[1] ^ w[2];
  return w[P];
}

// Walsh coefficients a_P of an odd b-bit table (codes 2^(b-1).. are the positive half).
__device__ __forceinline__ void walsh_coeffs(int bits, const float* c, float (&a)[4]) {
  a[0] = a[1] = a[2] = a[3] = 0.f;
  if (bits == 1) a[0] = c[1];
  if (bits == 2) { a[0] = 0.5f * (c[3] - c[2]); a[1] = 0.5f * (c[3] + c[2]); }
  if (bits == 3) {
    a[0] = 0.25f * (c[7] - c[6] + c[5] - c[4]);
    a[1] = 0.25f * (c[7] + c[6] - c[5] - c[4]);
    a[2] = 0.25f * (c[7] + c[6] + c[5] + c[4]);
    a[3] = 0.25f * (c[7] - c[6] - c[5] + c[4]);
  }
}

// Byte layout of one 32-token tile of a side with BITS code planes (and a sketch when QJL), as the
// host lays it out (kvq_api.cu make_side): planes, sketch words, fp16 norms, fp16 residual norms.
// Compile-time here so that every shared-memory address in the decode kernel is an immediate
// offset; launch_mma() refuses a cache whose runtime layout differs.
template <int BITS, bool QJL>
struct TileLayout {
  static constexpr int PLANES = 0;
  static constexpr int SKETCH = BITS * kTile * 16;
  static constexpr int NORM = SKETCH + (QJL ? kTile * 16 : 0);
  static constexpr int GAMMA = NORM + kTile * 2;
  static constexpr int BYTES = (GAMMA + (QJL ? kTile * 2 : 0) + 15) / 16 * 16;
  static bool matches(const SideLayout& L) {
    return L.off_planes == PLANES && L.off_sketch == SKETCH && L.off_norm == NORM &&
           (!QJL || L.off_gamma == GAMMA) && L.tile_bytes == BYTES && L.bits == BITS && L.qjl == QJL;
  }
};

// KIVI value tile: two code planes (byte-lane order), per-token fp16 scale (norm slot) and zero
// (gamma slot). KIVI key tiles are TileLayout<2, false> (their norm slot unused).
struct KiviVTile {
  static constexpr int PLANES = 0, SKETCH = 2 * kTile * 16, NORM = SKETCH, GAMMA = NORM + kTile * 2;
  static constexpr int BYTES = GAMMA + kTile * 2;
  static bool matches(const SideLayout& L) {
    return L.off_planes == PLANES && L.off_norm == NORM && L.off_gamma == GAMMA && L.tile_bytes == BYTES && L.bits == 2 &&
           !L.qjl;
  }
};
constexpr int kKiviStats = 2 * kHeadDim * 2;  // a key group's fp16 scales and zeros
constexpr int kKiviGroup = 128;               // tokens per KIVI key group

}  // namespace lmc
}  // namespace kvq
