// Prefill-rate LM / LM_QJL / SIGN1 quantize: one 32-token cache tile of one (sequence, kv-head,
// side) per block iteration, assembled in shared memory and written with 16-byte stores.
//
// Same per-vector computation as qlm::quantize_lm_block ("TurboQuant vs OSCAR vs EpiCache",
// section "Quantization frontiers: TurboQuant and OSCAR": random rotation, Lloyd-Max code per
// coordinate, 1-bit QJL sketch of the residual), organised for appends of many tokens:
//   * a warp codes 4 of the tile's tokens (norm, sign flip + FWHT, codes by ballot, residual);
//   * the sketch of all 32 residuals is one small product R [32 x 128] . S^T [128 x 128] with
//     S^T staged in shared memory once per block for all its tiles; thread (warp w, lane l) keeps
//     the projections of tokens 4w..4w+3 onto rows l + 32r, so one ballot per (token, r) is sign
//     word r of that token;
//   * the tile's bytes (code planes and sign words in the side's order, fp16 norms) are built in
//     shared memory -- with every token of an octet word present, no atomics -- and stored whole.
// A tile the call only partly covers (its first tokens were appended earlier, or the call ends
// inside it) is read first and only the call's tokens are replaced; a tile is owned by one block,
// so there is no race.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_quantize_lm.cuh"
#include "kvq_tiles.cuh"

namespace kvq {
namespace qtile {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxTileBytes = 3 * 512 + 512 + 128;  // planes + sketch + norms + gammas

// Shared memory: [S^T 128 x 128 floats] (sketch sides) | rho [32][128] | planes [32][3][4] |
// sign words [32][4] | norms, gammas [32] | tile bytes.
struct Smem {
  float rho[kTile][kHeadDim];
  uint32_t planes[kTile][kMaxBits][4];
  uint32_t z[kTile][4];
  float n[kTile], gamma[kTile];
  __align__(16) unsigned char tile[kMaxTileBytes];
};

inline size_t smem_bytes(bool sketch) { return sizeof(Smem) + (sketch ? sizeof(float) * kHeadDim * kHeadDim : 0); }

// Tiles per (sequence, head) the enumeration reserves: every call covers at most this many.
__host__ __device__ inline int max_tiles(int n_new) { return (n_new + 2 * kTile - 2) / kTile; }

__device__ __forceinline__ uint32_t spread_nibble(uint32_t x) {
  return (x & 1u) | ((x & 2u) << 7) | ((x & 4u) << 14) | ((x & 8u) << 21);
}

__device__ void quantize_tiles(const QuantizeParams& p, int side, float* st_s, Smem& sm) {
  const SideLayout& L = p.side[side];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int nthr = L.bits ? (1 << L.bits) - 1 : 0;
  const int tmax = max_tiles(p.n_new);
  const long total = (long)p.n_seq * p.heads * tmax;
  if (L.qjl && (long)blockIdx.x < total) {  // S^T once per block (cp.async, 16 B per thread per step)
    for (int c = tid; c < kHeadDim * kHeadDim / 4; c += kThreads) cp_async16(st_s + 4 * c, p.St + 4 * c);
    cp_async_commit();
  }
  float thr[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) thr[i] = i < nthr ? L.thr[i] : INFINITY;
  const float cent_lane = L.cent[(lane & 7) <= nthr ? (lane & 7) : 0];
  bool st_ready = false;

  for (long g = blockIdx.x; g < total; g += gridDim.x) {
    const int s = (int)(g / ((long)p.heads * tmax));
    const int h = (int)((g / tmax) % p.heads);
    const int k = (int)(g % tmax);
    const int pos0 = p.pos[s];
    const int tile = pos0 / kTile + k;
    const int t0 = tile * kTile;
    if (t0 >= pos0 + p.n_new) continue;  // the same for the whole block
    const int lo = max(t0, pos0) - t0, hi = min(t0 + kTile, pos0 + p.n_new) - t0;
    const long ti = tile_index(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.heads, p.seq[s], h, tile);
    if (ti < 0) {  // the block table names no page for this tile: nothing is written
      if (tid == 0) atomicOr(p.err, kStatusBadPage);
      continue;  // the same for the whole block
    }
    char* tb = p.region[side] + (size_t)ti * L.tile_bytes;
    // a tile whose first tokens are already stored: start from its current bytes
    if (lo > 0)
      for (int c = tid; c < L.tile_bytes / 16; c += kThreads)
        reinterpret_cast<uint4*>(sm.tile)[c] = reinterpret_cast<const uint4*>(tb)[c];

    // ---- per-token coding: warp w takes slots w, w + 8, w + 16, w + 24
    const float* sg = p.signs + h * p.signs_stride;
    float sgn[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) sgn[q] = sg[32 * q + lane];
#pragma unroll 1
    for (int slot = warp; slot < kTile; slot += kWarps) {
      if (slot < lo || slot >= hi) continue;
      // input rows of this (sequence, head): the call's n_new, or for window history the call's
      // src_rows, of which the history starts at row src_row0 - total0[s]
      const int rows = p.win_src ? p.src_rows : p.n_new, row0 = p.win_src ? p.src_row0 - p.total0[s] : 0;
      const size_t base = (((size_t)s * p.heads + h) * rows + (row0 + t0 + slot - pos0)) * kHeadDim;
      float u[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = qlm::load_elem(p.src[side], base + 32 * q + lane, p.bf16);
      const float n = sqrtf(qlm::warp_sum(u[0] * u[0] + u[1] * u[1] + u[2] * u[2] + u[3] * u[3]));
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] *= sgn[q];
#pragma unroll
      for (int b = 0; b < 5; ++b) {
        const bool upper = (lane >> b) & 1;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float other = __shfl_xor_sync(0xffffffffu, u[q], 1 << b);
          u[q] = upper ? other - u[q] : u[q] + other;
        }
      }
      const float a0 = u[0] + u[1], a1 = u[0] - u[1], a2 = u[2] + u[3], a3 = u[2] - u[3];
      u[0] = a0 + a2; u[2] = a0 - a2; u[1] = a1 + a3; u[3] = a1 - a3;
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = (n > 0.f) ? u[q] / n : 0.f;
      int code[4];
      float rho[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        int c = 0;
#pragma unroll
        for (int i = 0; i < 7; ++i) c += (u[q] >= thr[i]) ? 1 : 0;
        code[q] = c;
        rho[q] = u[q] - __shfl_sync(0xffffffffu, cent_lane, c);
      }
#pragma unroll
      for (int pp = 0; pp < kMaxBits; ++pp) {
        if (pp < L.bits) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t w = __ballot_sync(0xffffffffu, (code[q] >> pp) & 1);
            if (lane == q) sm.planes[slot][pp][q] = w;
          }
        }
      }
      if (L.qjl) {
#pragma unroll
        for (int q = 0; q < 4; ++q) sm.rho[slot][32 * q + lane] = rho[q];
        const float gam = sqrtf(qlm::warp_sum(rho[0] * rho[0] + rho[1] * rho[1] + rho[2] * rho[2] + rho[3] * rho[3]));
        if (lane == 0) sm.gamma[slot] = gam;
      }
      if (lane == 0) sm.n[slot] = n;
    }
    if (L.qjl && !st_ready) {
      cp_async_wait<0>();
      st_ready = true;
    }
    __syncthreads();

    // ---- sketch: projections of tokens 4w..4w+3 onto rows lane + 32 r
    if (L.qjl) {
      float acc[4][4];
#pragma unroll
      for (int v = 0; v < 4; ++v)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[v][r] = 0.f;
      const float* r0 = sm.rho[4 * warp];
#pragma unroll 4
      for (int i = 0; i < kHeadDim; i += 4) {
        float4 rv[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) rv[v] = *reinterpret_cast<const float4*>(r0 + v * kHeadDim + i);
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
          float sv[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) sv[r] = st_s[(i + ii) * kHeadDim + lane + 32 * r];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const float x = ii == 0 ? rv[v].x : ii == 1 ? rv[v].y : ii == 2 ? rv[v].z : rv[v].w;
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[v][r] = fmaf(sv[r], x, acc[v][r]);
          }
        }
      }
#pragma unroll
      for (int v = 0; v < 4; ++v)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t w = __ballot_sync(0xffffffffu, acc[v][r] >= 0.f);
          if (lane == r) sm.z[4 * warp + v][r] = w;
        }
      __syncthreads();
    }

    // ---- the tile's bytes, in the side's order
    const int nplanes = L.bits + (L.qjl ? 1 : 0);  // code planes, then the sign words
    auto word16 = [&](int slot, int pp, int q) -> uint32_t {  // word q of token `slot`'s 16-byte row
      return pp < L.bits ? sm.planes[slot][pp][q] : sm.z[slot][q];
    };
    auto plane_off = [&](int pp) { return pp < L.bits ? L.off_planes + pp * (kTile * 16) : L.off_sketch; };
    if (L.order == kOrderToken) {
      for (int idx = tid; idx < nplanes * kTile * 4; idx += kThreads) {
        const int pp = idx / (kTile * 4), slot = (idx / 4) % kTile, q = idx % 4;
        if (slot >= lo && slot < hi)
          *reinterpret_cast<uint32_t*>(sm.tile + plane_off(pp) + slot * 16 + 4 * q) = word16(slot, pp, q);
      }
    } else if (L.order == kOrderOctet) {
      // word x = 8t + 2m + hh of octet o: byte i is coordinate 32m + 16hh + 4t + i, bit j token 8o + j
      for (int idx = tid; idx < nplanes * 4 * 32; idx += kThreads) {
        const int pp = idx / 128, o = (idx / 32) % 4, x = idx % 32;
        if (8 * o + 7 < lo || 8 * o >= hi) continue;
        const int wt = x >> 3, wm = (x >> 1) & 3, wh = x & 1;
        uint32_t* dst = reinterpret_cast<uint32_t*>(sm.tile + plane_off(pp)) + o * 32 + x;
        uint32_t w = lo > 0 ? *dst : 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int slot = 8 * o + j;
          if (slot < lo || slot >= hi) continue;
          const uint32_t nib = (word16(slot, pp, wm) >> (16 * wh + 4 * wt)) & 0xFu;
          w = (w & ~(0x01010101u << j)) | (spread_nibble(nib) << j);
        }
        *dst = w;
      }
    } else {  // byte-lane-major: byte k of a token's 16-byte row goes to [k][slot]
      for (int idx = tid; idx < nplanes * 16 * kTile; idx += kThreads) {
        const int pp = idx / (16 * kTile), kk = (idx / kTile) % 16, slot = idx % kTile;
        if (slot >= lo && slot < hi)
          sm.tile[plane_off(pp) + kk * kTile + slot] = (unsigned char)((word16(slot, pp, kk >> 2) >> (8 * (kk & 3))) & 0xFFu);
      }
    }
    if (tid >= lo && tid < hi) {
      *reinterpret_cast<__half*>(sm.tile + L.off_norm + 2 * tid) = __float2half_rn(sm.n[tid]);
      if (L.qjl) *reinterpret_cast<__half*>(sm.tile + L.off_gamma + 2 * tid) = __float2half_rn(sm.gamma[tid]);
    }
    __syncthreads();
    for (int c = tid; c < L.tile_bytes / 16; c += kThreads)
      reinterpret_cast<uint4*>(tb)[c] = reinterpret_cast<const uint4*>(sm.tile)[c];
    __syncthreads();  // the next tile reuses the shared buffers
  }
  if (L.qjl && !st_ready) cp_async_wait<0>();
  if (side == 0 && blockIdx.x == 0)
    for (int i = tid; i < p.n_seq; i += kThreads) p.lens[p.seq[i]] = p.pos[i] + p.n_new;
}

}  // namespace qtile
}  // namespace kvq
