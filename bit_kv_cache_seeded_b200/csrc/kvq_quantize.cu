// Quantize-and-append kernels.
//
// LM / LM_QJL / SIGN1 ("TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers:
// TurboQuant and OSCAR"), one warp per vector, lane l holding coordinates 32k + l (k < 4):
//   1. n = ||x||                                    (warp sum of squares, fp32)
//   2. y = H D x                                    (sign flip; fast Walsh-Hadamard transform:
//                                                    5 shuffle stages over the lane bits and
//                                                    2 in-register stages over k)
//   3. u = y / n  (= sqrt(d) R x / n with R = H D / sqrt(d))
//   4. code_j = #{k : u_j >= t_k}                   (fp32 Lloyd-Max thresholds)
//   5. rho = u - c[code], gamma = ||rho||           (stage-two residual)
//   6. z_j = [ (S rho)_j >= 0 ]                     (1-bit QJL sketch, j < m)
//   7. one __ballot_sync per code plane / sketch word gives word k directly (bit l =
//      coordinate 32k + l), stored with one 16-byte store per plane; fp16 n and gamma.
//
// FP4 ("How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2", section "Numerics and
// hardware efficiency"): one warp per token, lane l owning the 16-channel group l:
//   s = E4M3_rn_satfinite(amax / 6); q_i = E2M1_rn_satfinite(x_i / s) (IEEE fp32 division);
//   a zero scale codes the group as zeros; RoPE key copied as bf16.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

__device__ __forceinline__ float load_elem(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr int kQuantWarps = 8;  // FP4 kernel: one token per warp
constexpr int kLmWarps = 4;     // LM kernel: warps per block

// LM quantize. Sides with a sketch: the block's 4 warps share one vector; each redoes steps 1-5
// (cheap, and it keeps every warp independent), then warp w forms sketch word w, i.e. the 32
// projections j = 32w + lane, from its own 16 KB column slice of S^T staged in shared memory.
// Sides without a sketch: one vector per warp.
__global__ void __launch_bounds__(kLmWarps * 32)
quantize_lm_kernel(const __grid_constant__ QuantizeParams p) {
  __shared__ float rho_s[kLmWarps][kHeadDim];
  extern __shared__ __align__(16) float st_s[];  // sketch sides: [warp][d][32] columns 32w.. of S^T
  const int side = blockIdx.y;
  const SideLayout& L = p.side[side];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthr = L.bits ? (1 << L.bits) - 1 : 0;
  const bool coop = L.qjl;
  const long total = (long)p.n_seq * p.heads * p.n_new;
  const long first = coop ? (long)blockIdx.x : (long)blockIdx.x * kLmWarps + warp;
  const long stride = coop ? (long)gridDim.x : (long)gridDim.x * kLmWarps;
  float* stw = st_s + warp * kHeadDim * 32;  // stw[i * 32 + l] = S^T[i][32 warp + l] = S[32 warp + l][i]
  // The slice is staged asynchronously while the first vector's elements are fetched.
  if (coop && first < total) {
    for (int c = lane; c < kHeadDim * 8; c += 32) {  // row i = c / 8, 16-byte chunk c % 8 of its 32 floats
      const int i = c >> 3, ch = c & 7;
      cp_async16(stw + i * 32 + ch * 4, p.St + (size_t)i * L.m + 32 * warp + ch * 4);
    }
    cp_async_commit();
  }
  float u_first[4] = {0.f, 0.f, 0.f, 0.f};
  if (first < total)
#pragma unroll
    for (int k = 0; k < 4; ++k) u_first[k] = load_elem(p.src[side], (size_t)first * kHeadDim + 32 * k + lane, p.bf16);
  if (coop) {
    cp_async_wait<0>();
    __syncwarp();
  }

  for (long vec = first; vec < total; vec += stride) {
    const int t = (int)(vec % p.n_new);
    const int h = (int)((vec / p.n_new) % p.heads);
    const int s = (int)(vec / ((long)p.n_new * p.heads));
    const size_t base = (size_t)vec * kHeadDim;  // [n_seq, heads, n_new, d] row-major

    float u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = (vec == first) ? u_first[k] : load_elem(p.src[side], base + 32 * k + lane, p.bf16);

    float n = 0.f;
    if (!p.skip_rotation) {
      n = sqrtf(warp_sum(u[0] * u[0] + u[1] * u[1] + u[2] * u[2] + u[3] * u[3]));
#pragma unroll
      for (int k = 0; k < 4; ++k) u[k] *= p.signs[32 * k + lane];
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
      for (int i = 0; i < nthr; ++i) c += (u[k] >= L.thr[i]) ? 1 : 0;
      code[k] = c;
      rho[k] = u[k] - L.cent[c];
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
      float proj = 0.f;  // (S rho)_j, j = 32 warp + lane
#pragma unroll 16
      for (int i = 0; i < kHeadDim; ++i) proj = fmaf(stw[i * 32 + lane], rho_s[warp][i], proj);
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
    char* tb = p.region[side] +
               (((size_t)seq * p.heads + h) * p.tiles_per_seq + tile) * (size_t)L.tile_bytes;
    if (L.tokmajor) {
      if (lead && lane < L.bits)
        *reinterpret_cast<uint4*>(tb + L.off_planes + lane * (kTile * 16) + slot * 16) = mine;
      if (coop && lane == 0) *reinterpret_cast<uint32_t*>(tb + L.off_sketch + slot * 16 + 4 * warp) = zword;
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

  if (side == 0 && blockIdx.x == 0 && !p.skip_rotation)
    for (int i = threadIdx.x; i < p.n_seq; i += blockDim.x) p.lens[p.seq[i]] = p.pos[i] + p.n_new;
}

// E2M1 code of an fp32 value: nearest grid point of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the
// even code, saturating at 6; the sign bit is kept even when the magnitude rounds to zero.
__device__ __forceinline__ uint32_t e2m1_code(float v) {
  const float a = fabsf(v);
  uint32_t c = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) +
               (a >= 3.5f) + (a > 5.0f);
  return c | (signbit(v) ? 8u : 0u);
}

__global__ void __launch_bounds__(kQuantWarps * 32)
quantize_fp4_kernel(const __grid_constant__ QuantizeParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const Fp4Layout& F = p.fp4;
  const long total = (long)p.n_seq * p.n_new;
  for (long tok = (long)blockIdx.x * kQuantWarps + warp; tok < total;
       tok += (long)gridDim.x * kQuantWarps) {
    const int t = (int)(tok % p.n_new);
    const int s = (int)(tok / p.n_new);
    const size_t lbase = (size_t)tok * F.latent + 16 * lane;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = load_elem(p.src[0], lbase + i, p.bf16);
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const __nv_fp8_storage_t sc = __nv_cvt_float_to_fp8(amax / 6.0f, __NV_SATFINITE, __NV_E4M3);
    const float scale = __half2float(__half(__nv_cvt_fp8_to_halfraw(sc, __NV_E4M3)));
    uint32_t lo = 0u, hi = 0u;
    if (scale > 0.f) {
#pragma unroll
      for (int i = 0; i < 8; ++i) lo |= e2m1_code(x[i] / scale) << (4 * i);
#pragma unroll
      for (int i = 0; i < 8; ++i) hi |= e2m1_code(x[8 + i] / scale) << (4 * i);
    }
    const int pos = p.pos[s] + t, seq = p.seq[s];
    const int tile = pos / kTile, slot = pos % kTile;
    char* tb = p.region[0] + ((size_t)seq * p.tiles_per_seq + tile) * (size_t)F.tile_bytes;
    *reinterpret_cast<uint2*>(tb + F.off_codes + slot * (F.latent / 2) + lane * 8) = make_uint2(lo, hi);
    tb[F.off_scales + slot * (F.latent / 16) + lane] = (char)sc;
    // RoPE key: rope bf16 values, 16 bytes per lane for the first rope/8 lanes.
    if (lane < F.rope / 8) {
      const size_t rbase = (size_t)tok * F.rope + 8 * lane;
      __nv_bfloat16 r[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) r[i] = __float2bfloat16_rn(load_elem(p.src[1], rbase + i, p.bf16));
      *reinterpret_cast<uint4*>(tb + F.off_rope + slot * (F.rope * 2) + lane * 16) =
          *reinterpret_cast<const uint4*>(r);
    }
  }
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.n_seq; i += blockDim.x) p.lens[p.seq[i]] = p.pos[i] + p.n_new;
}

int grid_for(long work_items, int per_block) {
  long blocks = (work_items + per_block - 1) / per_block;
  if (blocks > 148L * 16) blocks = 148L * 16;
  return blocks < 1 ? 1 : (int)blocks;
}

}  // namespace

cudaError_t launch_quantize_lm(const QuantizeParams& p, int n_sides, cudaStream_t s) {
  const long total = (long)p.n_seq * p.heads * p.n_new;
  const bool sketch = p.side[0].qjl || (n_sides > 1 && p.side[1].qjl);
  dim3 grid(grid_for(total, sketch ? 1 : kLmWarps), n_sides);  // sketch sides: one vector per block
  const size_t smem = sketch ? sizeof(float) * kHeadDim * kHeadDim : 0;  // m = d = 128
  cudaError_t e = cudaFuncSetAttribute(quantize_lm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  quantize_lm_kernel<<<grid, kLmWarps * 32, smem, s>>>(p);
  return launched();
}

cudaError_t launch_quantize_fp4(const QuantizeParams& p, cudaStream_t s) {
  const long total = (long)p.n_seq * p.n_new;
  quantize_fp4_kernel<<<grid_for(total, kQuantWarps), kQuantWarps * 32, 0, s>>>(p);
  return launched();
}

}  // namespace kvq
