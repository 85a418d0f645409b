// Mixed-precision window of an LM / LM_QJL / SIGN1 cache ("TurboQuant vs OSCAR vs EpiCache",
// section "Quantization frontiers: TurboQuant and OSCAR", OSCAR's mixed-precision paged memory: the
// sink tokens and the recent tokens stay in BF16 while the history in between is quantized).
//
// A sequence of T tokens keeps positions [0, min(T, sink)) in sink slots 0 .. sink - 1 and positions
// [max(sink, T - recent), T) in a ring of `recent` slots (position p in slot sink + (p - sink) % recent),
// as bf16 K and V; positions in between are coded into the cache's regular (history) region at
// history index p - sink. An append first codes the tokens that leave the window (from the ring, or
// straight from the input when the call appends more than the window holds), then writes the new
// tokens that stay in it (window_write, below). Decode runs the split kernels over the history and
// window_decode over the sink and recent tokens; the reduce merges the window's softmax state
// (m, l, o_r) with the splits'.
#include <cuda_bf16.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kWinThreads = 256;
constexpr int kWinMaxTokens = 1024;
constexpr int kWinMaxG = 8;
constexpr float kInvSqrtDw = 0.08838834764831845f;  // 1/sqrt(128)

__device__ __forceinline__ float load_in(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

// One warp per appended vector (sequence slot s, head h, token t); lane l moves coordinates 4l..4l+3.
__global__ void __launch_bounds__(kWinThreads) window_write(const __grid_constant__ QuantizeParams p) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long total = (long)p.n_seq * p.heads * p.n_new;
  for (long vec = (long)blockIdx.x * (kWinThreads / 32) + warp; vec < total;
       vec += (long)gridDim.x * (kWinThreads / 32)) {
    const int t = (int)(vec % p.n_new);
    const int h = (int)((vec / p.n_new) % p.heads);
    const int s = (int)(vec / ((long)p.n_new * p.heads));
    const int pos = p.total0[s] + t, end = p.total0[s] + p.n_new;
    int slot;
    if (pos < p.win_sink) slot = pos;
    else if (p.win_kivi && pos >= end - end % p.win_recent) slot = pos % p.win_recent;  // incomplete group
    else if (!p.win_kivi && p.win_recent > 0 && pos >= max(p.win_sink, end - p.win_recent))
      slot = p.win_sink + (pos - p.win_sink) % p.win_recent;
    else continue;  // this token was coded into the history
    const size_t in = (size_t)vec * kHeadDim + 4 * lane;
    const size_t out = (((size_t)p.seq[s] * p.heads + h) * p.win_slots + slot) * kHeadDim + 4 * lane;
#pragma unroll
    for (int side = 0; side < 2; ++side) {
      __nv_bfloat162 a = __floats2bfloat162_rn(load_in(p.src[side], in, p.bf16), load_in(p.src[side], in + 1, p.bf16));
      __nv_bfloat162 b = __floats2bfloat162_rn(load_in(p.src[side], in + 2, p.bf16), load_in(p.src[side], in + 3, p.bf16));
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&a);
      w.y = *reinterpret_cast<uint32_t*>(&b);
      *reinterpret_cast<uint2*>(const_cast<uint16_t*>(p.ring[side]) + out) = w;
    }
  }
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.n_seq; i += blockDim.x) p.lens[p.seq[i]] = p.total0[i] + p.n_new;
}

// One block per (kv-head, sequence): softmax state of every query head of the group over the sink and
// recent tokens, in the split kernels' partial format (logits in log2 units; o in the rotated domain,
// o_r = H D o / sqrt(d), so that the reduce's inverse rotation brings it back; no sketch part).
__global__ void __launch_bounds__(kWinThreads) window_decode(const __grid_constant__ DecodeParams p) {
  __shared__ __align__(16) float qs[kWinMaxG][kHeadDim];
  __shared__ float lg[kWinMaxG][kWinMaxTokens];
  __shared__ float stat[kWinMaxG][2];  // max, sum
  __shared__ float os[kWinMaxG][kHeadDim];
  const int hk = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = p.group;
  const int T = p.tot_lens[b];
  const int s_end = min(T, p.win_sink);
  const int r_begin = p.win_kivi ? T - T % p.win_recent : T > p.win_sink ? max(p.win_sink, T - p.win_recent) : s_end;
  const int n_sink = s_end, n_tok = s_end + (T - r_begin);
  auto slot_of = [&](int i) { return i < n_sink ? i : p.win_sink + (r_begin + (i - n_sink) - p.win_sink) % p.win_recent; };
  const size_t pair = (size_t)b * p.Hkv + hk;
  const uint16_t* kw = p.wk + pair * p.win_slots * kHeadDim;
  const uint16_t* vw = p.wv + pair * p.win_slots * kHeadDim;
  for (int i = tid; i < G * kHeadDim; i += kWinThreads) {
    const int h = i / kHeadDim, j = i % kHeadDim;
    qs[h][j] = load_in(p.q, ((size_t)b * p.Hq + hk * G + h) * kHeadDim + j, p.bf16) * p.logit_scale;
  }
  __syncthreads();
  // logits: token i by warp i % 8 (lane l: coordinates 4l .. 4l + 3), all heads, warp sums
  const int nw = kWinThreads / 32;
  constexpr int kBatch = 4;  // tokens per warp step: their key loads are in flight together
  for (int i0 = warp * kBatch; i0 < n_tok; i0 += nw * kBatch) {
    uint2 k4[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      k4[u] = i0 + u < n_tok ? *reinterpret_cast<const uint2*>(kw + (size_t)slot_of(i0 + u) * kHeadDim + 4 * lane)
                             : make_uint2(0u, 0u);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k4[u].x));
      const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&k4[u].y));
#pragma unroll
      for (int h = 0; h < kWinMaxG; ++h) {
        if (h >= G) break;
        const float4 q4 = *reinterpret_cast<const float4*>(&qs[h][4 * lane]);
        float v = fmaf(k23.y, q4.w, fmaf(k23.x, q4.z, fmaf(k01.y, q4.y, k01.x * q4.x)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && i0 + u < n_tok) lg[h][i0 + u] = v;
      }
    }
  }
  __syncthreads();
  // per head: max, then weights 2^(l - m) in place and their sum (warp h)
  if (warp < G) {
    float mx = -INFINITY;
    for (int i = lane; i < n_tok; i += 32) mx = fmaxf(mx, lg[warp][i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sm = 0.f;
    for (int i = lane; i < n_tok; i += 32) {
      const float w = exp2f(lg[warp][i] - mx);
      lg[warp][i] = w;
      sm += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
    if (lane == 0) { stat[warp][0] = mx; stat[warp][1] = sm; }
  }
  __syncthreads();
  // o[h][j] = sum_i w_i v_ij: thread (j, half) takes every other token and all heads, loading each
  // value element once; the two halves meet in shared memory. Signs applied (D o) for the rotation.
  {
    const int j = tid & (kHeadDim - 1), half = tid >> 7;
    float acc[kWinMaxG];
#pragma unroll
    for (int h = 0; h < kWinMaxG; ++h) acc[h] = 0.f;
    const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(vw);
    constexpr int kVBatch = 8;  // value loads in flight together
    for (int i0 = half; i0 < n_tok; i0 += 2 * kVBatch) {
      float v[kVBatch];
#pragma unroll
      for (int u = 0; u < kVBatch; ++u) {
        const int i = i0 + 2 * u;
        v[u] = i < n_tok ? __bfloat162float(vb[(size_t)slot_of(i) * kHeadDim + j]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kVBatch; ++u) {
        const int i = i0 + 2 * u;
        if (i < n_tok)
#pragma unroll
          for (int h = 0; h < kWinMaxG; ++h)
            if (h < G) acc[h] = fmaf(lg[h][i], v[u], acc[h]);
      }
    }
    if (half == 1)
#pragma unroll
      for (int h = 0; h < kWinMaxG; ++h)
        if (h < G) os[h][j] = acc[h];
    __syncthreads();
    const float* sg = p.signs + hk * p.signs_stride;
    if (half == 0)
#pragma unroll
      for (int h = 0; h < kWinMaxG; ++h)
        if (h < G) os[h][j] = p.win_kivi ? acc[h] + os[h][j] : (acc[h] + os[h][j]) * sg[j];
  }
  __syncthreads();
  if (p.win_kivi) {  // KIVI caches are not rotated: the state stays in the original domain
    for (int idx = tid; idx < G * kHeadDim; idx += kWinThreads) {
      const int h = idx / kHeadDim, j = idx % kHeadDim;
      p.wpart[((size_t)b * p.Hq + hk * G + h) * p.part_stride + 2 + j] = os[h][j];
    }
    if (tid < G) {
      float* dst = p.wpart + ((size_t)b * p.Hq + hk * G + tid) * p.part_stride;
      dst[0] = n_tok > 0 ? stat[tid][0] : -INFINITY;
      dst[1] = n_tok > 0 ? stat[tid][1] : 0.f;
    }
    return;
  }
  // o_r = H (D o) / sqrt(d): warp h, lane l holds coordinates 32k + l
  if (warp < G) {
    float u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = os[warp][32 * k + lane];
#pragma unroll
    for (int bb = 0; bb < 5; ++bb) {
      const bool upper = (lane >> bb) & 1;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float other = __shfl_xor_sync(0xffffffffu, u[k], 1 << bb);
        u[k] = upper ? other - u[k] : u[k] + other;
      }
    }
    const float a0 = u[0] + u[1], a1 = u[0] - u[1], a2 = u[2] + u[3], a3 = u[2] - u[3];
    u[0] = a0 + a2; u[2] = a0 - a2; u[1] = a1 + a3; u[3] = a1 - a3;
    float* dst = p.wpart + ((size_t)b * p.Hq + hk * G + warp) * p.part_stride;
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[2 + 32 * k + lane] = u[k] * kInvSqrtDw;
    if (p.v.qjl)
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[2 + kHeadDim + 32 * k + lane] = 0.f;
    if (lane == 0) {
      dst[0] = n_tok > 0 ? stat[warp][0] : -INFINITY;
      dst[1] = n_tok > 0 ? stat[warp][1] : 0.f;
    }
  }
}

}  // namespace

cudaError_t launch_window_write(const QuantizeParams& p, cudaStream_t s) {
  const long total = (long)p.n_seq * p.heads * p.n_new;
  long blocks = (total + kWinThreads / 32 - 1) / (kWinThreads / 32);
  if (blocks > 148L * 8) blocks = 148L * 8;
  window_write<<<(int)(blocks < 1 ? 1 : blocks), kWinThreads, 0, s>>>(p);
  return launched();
}

cudaError_t launch_window_decode(const DecodeParams& p, cudaStream_t s) {
  if (p.group > kWinMaxG || p.win_sink + p.win_recent > kWinMaxTokens) return cudaErrorNotSupported;
  window_decode<<<dim3(p.Hkv, p.B), kWinThreads, 0, s>>>(p);
  return launched();
}

}  // namespace kvq
