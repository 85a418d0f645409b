// Split-K decode attention over an FP4 MLA-style latent cache, and its split reduce.
//
// "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2": one 512-dim latent per token
// is shared by every head (section "CSA2") and stored as FP4 E2M1 with one scale per 16
// channels (section "Numerics and hardware efficiency"; the scale is an E4M3 byte here).
// With the absorbed query q = [q_lat ; q_rope]:
//   l_{h,t} = scale (q_lat[h] . latent_hat_t + q_rope[h] . k_rope_t)
//   out_h   = sum_t softmax_t(l_h) latent_hat_t
// latent_hat = E4M3 scale x E2M1 value, exact in fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kMlaThreads = 256;
constexpr int kLat = 512, kRope = 64, kLatPad = kLat + 1, kRopePad = kRope + 1;

__device__ __forceinline__ float exp2_diff(float a, float b) {
  return (a == -INFINITY) ? 0.f : exp2f(a - b);
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float e2m1_value(uint32_t nib) {
  const uint32_t m = nib & 7u;
  // grid {0, .5, 1, 1.5, 2, 3, 4, 6}: exponent field m>>1, mantissa bit m&1 (bias 1)
  const float mag = (m < 2u) ? 0.5f * (float)m : (float)(1u << ((m >> 1) - 1)) * (1.f + 0.5f * (float)(m & 1u));
  return (nib & 8u) ? -mag : mag;
}

__device__ __forceinline__ float e4m3_value(uint8_t byte) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)byte, __NV_E4M3)));
}

__device__ __forceinline__ float load_q(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

template <int HPW>  // heads per warp (8 warps)
__global__ void __launch_bounds__(kMlaThreads)
decode_mla_simple(const __grid_constant__ MlaParams p) {
  extern __shared__ float sm[];
  float* lat_s = sm;                              // [32][kLatPad]
  float* rope_s = lat_s + kTile * kLatPad;        // [32][kRopePad]
  float* q_s = rope_s + kTile * kRopePad;         // [Hq][576]
  const int split = blockIdx.x, b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int Hq = p.Hq;
  const int len = p.lens[b];
  const int t_begin = split * p.chunk;
  const int t_end = min(len, t_begin + p.chunk);
  const int dq = kLat + kRope;

  for (int idx = threadIdx.x; idx < Hq * dq; idx += kMlaThreads)
    q_s[idx] = load_q(p.q, (size_t)b * Hq * dq + idx, p.bf16) * p.logit_scale;

  float m_run[HPW], l_run[HPW], o[HPW][16];
#pragma unroll
  for (int i = 0; i < HPW; ++i) {
    m_run[i] = -INFINITY;
    l_run[i] = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) o[i][k] = 0.f;
  }
  const Fp4Layout& F = p.fp4;
  for (int tile = t_begin / kTile; tile * kTile < t_end; ++tile) {
    const int count = min(kTile, t_end - tile * kTile);
    const char* tb = p.reg + ((size_t)b * p.tiles_per_seq + tile) * (size_t)F.tile_bytes;
    __syncthreads();
    for (int idx = threadIdx.x; idx < kTile * kLat; idx += kMlaThreads) {
      const int t = idx / kLat, c = idx % kLat;
      float v = 0.f;
      if (t < count) {
        const uint8_t byte = (uint8_t)tb[F.off_codes + t * (kLat / 2) + c / 2];
        const uint8_t sc = (uint8_t)tb[F.off_scales + t * (kLat / 16) + c / 16];
        v = e4m3_value(sc) * e2m1_value((byte >> (4 * (c & 1))) & 0xF);
      }
      lat_s[t * kLatPad + c] = v;
    }
    for (int idx = threadIdx.x; idx < kTile * kRope; idx += kMlaThreads) {
      const int t = idx / kRope, r = idx % kRope;
      float v = 0.f;
      if (t < count) v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(tb + F.off_rope)[t * kRope + r]);
      rope_s[t * kRopePad + r] = v;
    }
    __syncthreads();
    const bool valid = lane < count;
    float pr[HPW];
#pragma unroll
    for (int i = 0; i < HPW; ++i) {
      const int h = warp + 8 * i;
      const float* qh = q_s + h * dq;
      float acc = 0.f;
      for (int c = 0; c < kLat; ++c) acc = fmaf(qh[c], lat_s[lane * kLatPad + c], acc);
      for (int r = 0; r < kRope; ++r) acc = fmaf(qh[kLat + r], rope_s[lane * kRopePad + r], acc);
      const float lg = valid ? acc : -INFINITY;
      const float m_new = fmaxf(m_run[i], warp_max(lg));
      const float corr = exp2_diff(m_run[i], m_new);
      pr[i] = exp2_diff(lg, m_new);
      l_run[i] = l_run[i] * corr + warp_sum(pr[i]);
      m_run[i] = m_new;
#pragma unroll
      for (int k = 0; k < 16; ++k) o[i][k] *= corr;
    }
    for (int t = 0; t < count; ++t) {
      float lv[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) lv[k] = lat_s[t * kLatPad + lane + 32 * k];
#pragma unroll
      for (int i = 0; i < HPW; ++i) {
        const float pt = __shfl_sync(0xffffffffu, pr[i], t);
#pragma unroll
        for (int k = 0; k < 16; ++k) o[i][k] = fmaf(pt, lv[k], o[i][k]);
      }
    }
  }
  const int stride = 2 + kLat;
#pragma unroll
  for (int i = 0; i < HPW; ++i) {
    const int h = warp + 8 * i;
    float* dst = p.part + (((size_t)b * Hq + h) * p.splits + split) * stride;
    if (lane == 0) { dst[0] = m_run[i]; dst[1] = l_run[i]; }
#pragma unroll
    for (int k = 0; k < 16; ++k) dst[2 + lane + 32 * k] = o[i][k];
  }
}

// Merge of a row's split partials (log-sum-exp): block (row, quarter) takes latent channels
// 128 quarter .. + 127. The splits' maximum and their weights 2^(m_s - M) are formed once per block
// (threads over splits, a fixed reduction order) and staged in shared memory, kRedChunk splits at a
// time; thread (group g, channel) then sums its channel over the splits s = g mod 4 (reading them
// coalesced, several loads in flight) and the four groups' sums are added in a fixed order.
constexpr int kRedChannels = 128, kRedGroups = 4, kRedThreads = kRedChannels * kRedGroups, kRedChunk = 512;

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, x) : v + x;
  }
  __syncthreads();  // sh may still be read from the previous reduction
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  float r = sh[0];
#pragma unroll
  for (int w = 1; w < kRedThreads / 32; ++w) r = is_max ? fmaxf(r, sh[w]) : r + sh[w];
  return r;
}

__global__ void __launch_bounds__(kRedThreads) reduce_mla(const __grid_constant__ MlaParams p) {
  __shared__ float s_w[kRedChunk];
  __shared__ float s_red[kRedThreads / 32];
  __shared__ float s_o[kRedGroups][kRedChannels];
  const int row = blockIdx.x / (kLat / kRedChannels), tid = threadIdx.x;
  const int grp = tid / kRedChannels, c = (blockIdx.x % (kLat / kRedChannels)) * kRedChannels + tid % kRedChannels;
  const int stride = 2 + kLat;
  const float* part = p.part + (size_t)row * p.splits * stride;
  float m = -INFINITY;
  for (int sp = tid; sp < p.splits; sp += kRedThreads) m = fmaxf(m, part[(size_t)sp * stride]);
  const float M = block_reduce(m, true, s_red);
  float l = 0.f, o = 0.f;
  for (int s0 = 0; s0 < p.splits; s0 += kRedChunk) {
    const int n = min(kRedChunk, p.splits - s0);
    __syncthreads();  // the previous chunk's weights have been used
    for (int i = tid; i < n; i += kRedThreads) {
      const float* ps = part + (size_t)(s0 + i) * stride;
      const float w = exp2_diff(ps[0], M);
      s_w[i] = w;
      l += w * ps[1];
    }
    __syncthreads();
    const float* pc = part + (size_t)s0 * stride + 2 + c;
#pragma unroll 8
    for (int i = grp; i < n; i += kRedGroups) o = fmaf(s_w[i], pc[(size_t)i * stride], o);
  }
  const float L = block_reduce(l, false, s_red);
  s_o[grp][tid % kRedChannels] = o;
  __syncthreads();
  if (grp != 0) return;
  o = (s_o[0][tid] + s_o[1][tid]) + (s_o[2][tid] + s_o[3][tid]);
  if (p.pout) {  // merged softmax state: running maximum (log2 units), sum of weights, unnormalised o
    float* st = p.pout + (size_t)row * stride;
    st[2 + c] = o;
    if (c == 0) {
      st[0] = M;
      st[1] = L;
    }
    return;
  }
  p.out[(size_t)row * kLat + c] = (L > 0.f) ? o / L : 0.f;
}

size_t mla_smem_bytes(int Hq) {
  return sizeof(float) * ((size_t)kTile * kLatPad + (size_t)kTile * kRopePad + (size_t)Hq * (kLat + kRope));
}

template <int HPW>
cudaError_t launch_hpw(const MlaParams& p, cudaStream_t s) {
  const size_t smem = mla_smem_bytes(p.Hq);
  cudaError_t e = cudaFuncSetAttribute(decode_mla_simple<HPW>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_mla_simple<HPW><<<dim3(p.splits, p.B), kMlaThreads, smem, s>>>(p);
  return launched();
}

}  // namespace

cudaError_t launch_decode_mla(const MlaParams& p, cudaStream_t s) {
  if (mla_umma_supported(p)) return launch_decode_mla_umma(p, s);  // 64 heads: tcgen05
  if (mla_mma_supported(p)) return launch_decode_mla_mma(p, s);
  if (p.fp4.latent != kLat || p.fp4.rope != kRope) return cudaErrorNotSupported;
  switch (p.Hq) {
    case 8: return launch_hpw<1>(p, s);
    case 16: return launch_hpw<2>(p, s);
    case 32: return launch_hpw<4>(p, s);
    case 64: return launch_hpw<8>(p, s);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_reduce_mla(const MlaParams& p, cudaStream_t s) {
  reduce_mla<<<p.B * p.Hq * (kLat / kRedChannels), kRedThreads, 0, s>>>(p);
  return launched();
}

}  // namespace kvq
