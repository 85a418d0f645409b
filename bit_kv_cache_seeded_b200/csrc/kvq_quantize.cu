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
#include <algorithm>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_quantize_lm.cuh"
#include "kvq_quantize_tile.cuh"

namespace kvq {
namespace {

constexpr int kQuantWarps = 8;  // FP4 kernel: one token per warp
constexpr int kTileQuantizeMinTokens = 16;  // appends of at least this many tokens per sequence use the tile kernel
using qlm::kLmWarps;
using qlm::load_elem;

// LM quantize: grid (blocks, sides); the work of one block is qlm::quantize_lm_block.
__global__ void __launch_bounds__(qlm::kLmWarps * 32)
quantize_lm_kernel(const __grid_constant__ QuantizeParams p) {
  qlm::quantize_lm_block(p, blockIdx.y, blockIdx.x, gridDim.x);
}

// Prefill-rate LM quantize: grid (blocks, sides); tiles of one side per block (kvq_quantize_tile.cuh).
__global__ void __launch_bounds__(qtile::kThreads)
quantize_lm_tile_kernel(const __grid_constant__ QuantizeParams p) {
  extern __shared__ __align__(16) unsigned char qt_smem[];
  const bool sketch = p.side[0].qjl || p.side[1].qjl;
  qtile::Smem& sm = *reinterpret_cast<qtile::Smem*>(qt_smem);
  float* st_s = reinterpret_cast<float*>(qt_smem + sizeof(qtile::Smem));
  qtile::quantize_tiles(p, blockIdx.y, sketch ? st_s : nullptr, sm);
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
  if (n_sides == 2 && !p.skip_rotation && (!p.win_src || p.win_input_only) && p.n_new >= kTileQuantizeMinTokens) {
    // appends of many tokens per sequence: whole tiles per block, 16-byte stores, S^T staged once
    const bool sketch = p.side[0].qjl || p.side[1].qjl;
    const long tiles = (long)p.n_seq * p.heads * qtile::max_tiles(p.n_new);
    const size_t smem = qtile::smem_bytes(sketch);
    cudaError_t e = cudaFuncSetAttribute(quantize_lm_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int blocks = (int)std::min<long>(tiles, 148L * 2);
    quantize_lm_tile_kernel<<<dim3(blocks, 2), qtile::kThreads, smem, s>>>(p);
    return launched();
  }
  QuantizeParams q = p;
  if (n_sides < 2) q.side[1] = q.side[0];  // the block count looks at both sides
  const bool sketch = p.side[0].qjl || (n_sides > 1 && p.side[1].qjl);
  dim3 grid(qlm::blocks_per_side(q), n_sides);
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
