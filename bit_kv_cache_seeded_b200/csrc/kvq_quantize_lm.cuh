// LM / LM_QJL / SIGN1 quantize-and-append, as a block-level device function so that it can run
// alone (quantize_lm_kernel) or beside the query prep of a fused decode step (one launch).
//
// "TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and OSCAR"; the
// steps are listed at the top of kvq_quantize.cu.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_tiles.cuh"

namespace kvq {
namespace qlm {

__device__ __forceinline__ float load_elem(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kLmWarps = 4;     // LM quantize: warps per block

// Where vector t of sequence slot s, head h of an LM quantize call starts, and whether it is bf16.
// Plain calls: row t of the [n_seq, heads, n_new, d] input. History appends of a window cache: the
// token at sequence position sink + pos[s] + t, from the bf16 ring below the old length, else from
// the input (rows of src_rows per (sequence, head)).
__device__ __forceinline__ const void* vector_src(const QuantizeParams& p, int side, int s, int h, int t, int& bf16) {
  bf16 = p.bf16;
  if (!p.win_src) {
    const size_t elem = p.bf16 ? 2 : 4;
    return static_cast<const char*>(p.src[side]) + ((((size_t)s * p.heads + h) * p.n_new + t) * kHeadDim) * elem;
  }
  const int pos = p.win_sink + p.pos[s] + t;
  if (pos < p.total0[s]) {
    bf16 = 1;
    const int slot = p.win_sink + (pos - p.win_sink) % p.win_recent;
    return p.ring[side] + (((size_t)p.seq[s] * p.heads + h) * p.win_slots + slot) * kHeadDim;
  }
  const size_t elem = p.bf16 ? 2 : 4;
  return static_cast<const char*>(p.src[side]) +
         ((((size_t)s * p.heads + h) * p.src_rows + (pos - p.total0[s])) * kHeadDim) * elem;
}

// Bits 0..3 of x moved to bits 0, 8, 16, 24.
__device__ __forceinline__ uint32_t spread_nibble(uint32_t x) {
  return (x & 1u) | ((x & 2u) << 7) | ((x & 4u) << 14) | ((x & 8u) << 21);
}

// Blocks per side of an LM quantize launch: one vector per block on sides with a sketch (the
// block's warps share it), one per warp otherwise; at most 16 blocks per SM of a B200.
inline int blocks_per_side(const QuantizeParams& p) {
  const long total = (long)p.n_seq * p.heads * p.n_new;
  const bool sketch = p.side[0].qjl || p.side[1].qjl;
  const long per = sketch ? 1 : kLmWarps;
  long blocks = (total + per - 1) / per;
  if (blocks > 148L * 16) blocks = 148L * 16;
  return blocks < 1 ? 1 : (int)blocks;
}

// One block of the LM quantize (`blk` of `nblk` blocks of side `side`). Sides with a sketch: the
// block's 4 warps share one vector; each redoes steps 1-5 (cheap, and it keeps every warp
// independent), then warp w forms sketch word w, i.e. the 32 projections j = 32w + lane, from
// columns 32w.. of S^T, which one bulk copy brings into shared memory while steps 1-5 run.
// Sides without a sketch: one vector per warp.
__device__ __forceinline__ void quantize_lm_block(const QuantizeParams& p, int side, int blk, int nblk) {
  __shared__ __align__(16) float rho_s[kLmWarps][kHeadDim];
  __shared__ __align__(8) uint64_t st_bar;       // completes when S^T has landed
  extern __shared__ __align__(16) float st_s[];  // sketch sides: S^T [d][m], m = d = 128
  const SideLayout& L = p.side[side];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthr = L.bits ? (1 << L.bits) - 1 : 0;
  const bool coop = L.qjl;
  const long total = (long)p.n_seq * p.heads * p.n_new;
  const long first = coop ? (long)blk : (long)blk * kLmWarps + warp;
  const long stride = coop ? (long)nblk : (long)nblk * kLmWarps;
  const bool staged = coop && first < total;  // the same for every thread of the block
  bool st_failed = false;
  if (staged) {
    if (threadIdx.x == 0) {
      const uint32_t bar = smem_addr(&st_bar);
      mbar_init(bar, 1);
      mbar_init_fence();
      constexpr uint32_t kQuarter = kHeadDim * kHeadDim / 4;  // floats in a quarter of S^T (16 KB)
      mbar_arrive_expect_tx(bar, 4u * kQuarter * 4u);
#pragma unroll
      for (int c = 0; c < 4; ++c) bulk_g2s(smem_addr(st_s + c * kQuarter), p.St + c * kQuarter, kQuarter * 4u, bar);
    }
    // no block barrier here: the one before the first wait below publishes the initialisation
  }
  const float* stw = st_s + 32 * warp + lane;  // stw[i * d] = S^T[i][32 warp + lane] = S[32 warp + lane][i]
  // Everything the first vector needs from global memory is requested before the staged slice
  // is waited for (which happens only right before the sketch product).
  // Launched as a programmatic dependent (fused decode step): everything above reads only the
  // cache's own constants; the inputs may come from the preceding kernel, so wait for it here.
  grid_dep_wait();
  float u_first[4] = {0.f, 0.f, 0.f, 0.f};
  if (first < total && !p.win_src)
#pragma unroll
    for (int k = 0; k < 4; ++k) u_first[k] = load_elem(p.src[side], (size_t)first * kHeadDim + 32 * k + lane, p.bf16);
  bool block_synced = false;  // the block barrier before the first wait for S^T has been passed
  float sg[4];  // rotation signs (the debug entry's inputs are already rotated: none read)
  int sg_head = 0;  // the head whose diagonal sg holds (per-head rotation)
  if (first < total) sg_head = (int)((first / p.n_new) % p.heads);
#pragma unroll
  for (int k = 0; k < 4; ++k) sg[k] = p.skip_rotation ? 1.f : p.signs[sg_head * p.signs_stride + 32 * k + lane];
  // the table in registers: thresholds (unused ones +inf), centroid c held by lane c % 8
  float thr[7];
#pragma unroll
  for (int i = 0; i < 7; ++i) thr[i] = i < nthr ? L.thr[i] : INFINITY;
  const float cent_lane = L.cent[(lane & 7) <= nthr ? (lane & 7) : 0];

  for (long vec = first; vec < total; vec += stride) {
    const int t = (int)(vec % p.n_new);
    const int h = (int)((vec / p.n_new) % p.heads);
    const int s = (int)(vec / ((long)p.n_new * p.heads));
    if (p.win_src && t >= p.cnt[s]) continue;  // uniform over the vector's warp (block: coop sides)

    float u[4];
    if (vec == first && !p.win_src) {
#pragma unroll
      for (int k = 0; k < 4; ++k) u[k] = u_first[k];
    } else {
      int vb16;
      const void* src = vector_src(p, side, s, h, t, vb16);
#pragma unroll
      for (int k = 0; k < 4; ++k) u[k] = load_elem(src, 32 * k + lane, vb16);
    }

    if (p.signs_stride && h != sg_head && !p.skip_rotation) {  // per-head rotation: this head's diagonal
      sg_head = h;
#pragma unroll
      for (int k = 0; k < 4; ++k) sg[k] = p.signs[h * p.signs_stride + 32 * k + lane];
    }
    float n = 0.f;
    if (!p.skip_rotation) {
      n = sqrtf(warp_sum(u[0] * u[0] + u[1] * u[1] + u[2] * u[2] + u[3] * u[3]));
#pragma unroll
      for (int k = 0; k < 4; ++k) u[k] *= sg[k];
      // Walsh-Hadamard butterflies over index bits 0..4 (lane) and 5..6 (k).
#pragma unroll
      for (int b = 0; b < 5; ++b) {
        const bool upper = (lane >> b) & 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float other = __shfl_xor_sync(0xffffffffu, u[k], 1 << b);
          u[k] = upper ? other - u[k] : u[k] + other;
        }
      }
      const float a0 = u[0] + u[1], a1 = u[0] - u[1], a2 = u[2] + u[3], a3 = u[2] - u[3];
      u[0] = a0 + a2; u[2] = a0 - a2; u[1] = a1 + a3; u[3] = a1 - a3;
#pragma unroll
      for (int k = 0; k < 4; ++k) u[k] = (n > 0.f) ? u[k] / n : 0.f;
    }

    int code[4];
    float rho[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int c = 0;
#pragma unroll
      for (int i = 0; i < 7; ++i) c += (u[k] >= thr[i]) ? 1 : 0;
      code[k] = c;
      rho[k] = u[k] - __shfl_sync(0xffffffffu, cent_lane, c);
    }
    uint32_t planes[kMaxBits][4];
#pragma unroll
    for (int pp = 0; pp < kMaxBits; ++pp)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        planes[pp][k] = (pp < L.bits) ? __ballot_sync(0xffffffffu, (code[k] >> pp) & 1) : 0u;
    // lane pp < bits stores plane pp (selected without indexing registers by lane)
    uint4 mine = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int pp = 0; pp < kMaxBits; ++pp)
      if (lane == pp) mine = make_uint4(planes[pp][0], planes[pp][1], planes[pp][2], planes[pp][3]);

    uint32_t zword = 0u;  // sketch word `warp` (coop sides)
    float gamma = 0.f;
    if (coop) {
      gamma = sqrtf(warp_sum(rho[0] * rho[0] + rho[1] * rho[1] + rho[2] * rho[2] + rho[3] * rho[3]));
#pragma unroll
      for (int k = 0; k < 4; ++k) rho_s[warp][32 * k + lane] = rho[k];
      __syncwarp();
      if (!block_synced) {
        __syncthreads();  // st_bar was initialised (by thread 0) before anyone waits
        if (!mbar_try(smem_addr(&st_bar), 0u) && !mbar_wait(smem_addr(&st_bar), 0u, p.wait_limit)) {
          st_failed = true;  // S^T (requested at the start)
          atomicOr(p.err, 1);
        }
        block_synced = true;
      }
      __syncwarp();
      float pr[4] = {0.f, 0.f, 0.f, 0.f};  // (S rho)_j, j = 32 warp + lane: four partial chains
#pragma unroll 8
      for (int i = 0; i < kHeadDim; i += 4) {
        const float4 r = *reinterpret_cast<const float4*>(&rho_s[warp][i]);
        pr[0] = fmaf(stw[i * kHeadDim], r.x, pr[0]);
        pr[1] = fmaf(stw[(i + 1) * kHeadDim], r.y, pr[1]);
        pr[2] = fmaf(stw[(i + 2) * kHeadDim], r.z, pr[2]);
        pr[3] = fmaf(stw[(i + 3) * kHeadDim], r.w, pr[3]);
      }
      const float proj = (pr[0] + pr[1]) + (pr[2] + pr[3]);
      __syncwarp();
      zword = __ballot_sync(0xffffffffu, proj >= 0.f);
    }
    const bool lead = !coop || warp == 0;  // writes the planes and norms of this vector

    if (p.skip_rotation) {
      if (lead && lane < L.bits)
        *reinterpret_cast<uint4*>(p.dbg_planes + ((size_t)vec * L.bits + lane) * 4) = mine;
      if (coop && lane == 0) p.dbg_sketch[(size_t)vec * 4 + warp] = zword;
      if (coop && warp == 0 && lane == 1) p.dbg_gamma[vec] = __half_as_ushort(__float2half_rn(gamma));
      continue;
    }

    const int pos = p.pos[s] + t;
    const int seq = p.seq[s];
    const int tile = pos / kTile, slot = pos % kTile;
    const long ti = tile_index(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.heads, seq, h, tile);
    if (ti < 0) {  // the block table names no page for this token: nothing is written
      if (threadIdx.x % 32 == 0) atomicOr(p.err, kStatusBadPage);
      continue;
    }
    char* tb = p.region[side] + (size_t)ti * L.tile_bytes;
    if (L.order == kOrderToken) {
      if (lead && lane < L.bits)
        *reinterpret_cast<uint4*>(tb + L.off_planes + lane * (kTile * 16) + slot * 16) = mine;
      if (coop && lane == 0) *reinterpret_cast<uint32_t*>(tb + L.off_sketch + slot * 16 + 4 * warp) = zword;
    } else if (L.order == kOrderOctet) {
      // bit (slot % 8) of each byte of word x = 8t + 2m + h of octet slot / 8; byte i of the word
      // is coordinate 32m + 16h + 4t + i. Neighbouring tokens share the words, so this token's bits
      // are cleared and set with atomics (other tokens' bits are never touched).
      const uint32_t jmask = 0x01010101u << (slot & 7);
      uint32_t* octet = reinterpret_cast<uint32_t*>(tb) + (slot >> 3) * 32;
      if (lead) {  // lane = word x of every plane
        const int wt = lane >> 3, wm = (lane >> 1) & 3, wh = lane & 1;
#pragma unroll
        for (int pp = 0; pp < kMaxBits; ++pp) {
          if (pp < L.bits) {
            const uint32_t src = wm == 0 ? planes[pp][0] : wm == 1 ? planes[pp][1] : wm == 2 ? planes[pp][2] : planes[pp][3];
            const uint32_t bits4 = (src >> (16 * wh + 4 * wt)) & 0xFu;
            uint32_t* w = octet + (L.off_planes + pp * (kTile * 16)) / 4 + lane;
            atomicAnd(w, ~jmask);
            atomicOr(w, spread_nibble(bits4) << (slot & 7));
          }
        }
      }
      if (coop && lane < 8) {  // sign word `warp` is coordinate block m = warp: words 8t + 2 warp + h
        const int wt = lane >> 1, wh = lane & 1;
        const uint32_t bits4 = (zword >> (16 * wh + 4 * wt)) & 0xFu;
        uint32_t* w = octet + L.off_sketch / 4 + 8 * wt + 2 * warp + wh;
        atomicAnd(w, ~jmask);
        atomicOr(w, spread_nibble(bits4) << (slot & 7));
      }
    } else {
      // byte-lane-major: byte k of a token's 16-byte plane goes to [k][slot]
      if (lead && lane < 16) {
#pragma unroll
        for (int pp = 0; pp < kMaxBits; ++pp) {
          if (pp < L.bits) {  // byte `lane` of plane pp: word lane / 4, byte lane % 4
            const uint32_t lo = (lane & 4) ? planes[pp][1] : planes[pp][0];
            const uint32_t hi = (lane & 4) ? planes[pp][3] : planes[pp][2];
            const uint32_t w = (lane & 8) ? hi : lo;
            tb[L.off_planes + pp * (kTile * 16) + lane * kTile + slot] = (char)((w >> (8 * (lane & 3))) & 0xFFu);
          }
        }
      }
      if (coop && lane < 4)
        tb[L.off_sketch + (4 * warp + lane) * kTile + slot] = (char)((zword >> (8 * lane)) & 0xFFu);
    }
    if (lead && lane == 30) *reinterpret_cast<__half*>(tb + L.off_norm + slot * 2) = __float2half_rn(n);
    if (coop && warp == 0 && lane == 29)
      *reinterpret_cast<__half*>(tb + L.off_gamma + slot * 2) = __float2half_rn(gamma);
  }

  // a wait that gave up: the copy may still be landing, so wait for it (bounded) before leaving; a
  // staged block whose vectors were all skipped still waits for its copy
  if (st_failed || (staged && !block_synced && threadIdx.x == 0)) mbar_wait(smem_addr(&st_bar), 0u, p.wait_limit);
  if (side == 0 && blk == 0 && !p.skip_rotation)
    for (int i = threadIdx.x; i < p.n_seq; i += blockDim.x)
      p.lens[p.seq[i]] = p.pos[i] + (p.win_src ? p.cnt[i] : p.n_new);
}

}  // namespace qlm
}  // namespace kvq
