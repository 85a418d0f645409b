// Decode over the mixed-precision window ("TurboQuant vs OSCAR vs EpiCache", section "Quantization
// frontiers: TurboQuant and OSCAR": sink and recent tokens kept in BF16 beside the coded history),
// as a CTA-wide device function: the standalone window kernel and the mma.sync split kernel's extra
// CTAs both run it.
//
// The window of a sequence with T tokens occupies a prefix of its slots: sink slots [0, min(T, sink))
// and, once T > sink, ring slots sink .. sink + min(recent, T - sink) - 1 (a KIVI cache: the
// incomplete last key group, slots [0, T % 128)). Softmax does not depend on the order of its terms,
// so the window is read slot by slot, and every part of kWinPart slots is one contiguous run of K and
// V rows. A part yields the softmax state (m, l, o) of its tokens in the split kernels' partial format
// (logits in log2 units; o rotated, o_r = H D o / sqrt(d), on rotated caches); the reduce merges the
// parts with the splits.
#pragma once
#include <cuda_bf16.h>

#include "kvq_internal.h"

namespace kvq {

constexpr int kWinPart = 64;  // window slots per part (one CTA)

__host__ __device__ constexpr int window_parts(int slots) { return (slots + kWinPart - 1) / kWinPart; }

// Shared floats window_part<NW, GH> uses: query, logits / weights, per-group value sums, (m, l).
template <int NW, int GH>
__host__ __device__ constexpr int window_smem_floats() {
  return GH * (kHeadDim + kWinPart + (NW / 2) * kHeadDim + 2);
}

// Window tokens of a sequence with T tokens (they fill slots [0, n)).
__device__ __forceinline__ int window_tokens(const DecodeParams& p, int T) {
  if (p.win_kivi) return T % p.win_recent;
  const int ns = min(T, p.win_sink);
  const int nr = T > p.win_sink ? min(p.win_recent, T - p.win_sink) : 0;
  return ns + nr;
}

// Softmax state of query heads hk * group + h0 .. + GH - 1 of sequence b over window part `part`, by
// a CTA of NW warps (sm: window_smem_floats<NW, GH>() floats of shared memory). Rows are loaded in
// small batches with the next batch in flight, so the path needs few registers (it also runs inside
// the split kernel, whose register count it must not raise).
template <int NW, int GH>
__device__ __forceinline__ void window_part(const DecodeParams& p, int b, int hk, int h0, int part, float* sm) {
  static_assert(NW == 4 || NW == 8, "four or eight warps");
  constexpr int NT = NW * 32;
  constexpr int TPW = kWinPart / NW;      // key rows per warp (16 or 8)
  constexpr int NG = NW / 2;              // value row groups: thread (c2, tg) takes columns 2 c2, 2 c2 + 1
  constexpr int TPG = kWinPart / NG;      // value rows per group
  float* qs = sm;                         // [GH][d] query, in log2 logit units
  float* lg = qs + GH * kHeadDim;         // [GH][kWinPart] logits, then weights
  float* red = lg + GH * kWinPart;        // [NG][GH][d] value sums per row group
  float* stat = red + NG * GH * kHeadDim; // [GH][2] max, sum
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = window_tokens(p, __ldcg(p.tot_lens + b));
  const int t0 = part * kWinPart;
  const int cnt = min(kWinPart, n - t0);  // tokens of this part (<= 0: none)
  const int hq0 = hk * p.group + h0;
  const size_t hstride = (size_t)p.win_parts * p.part_stride;
  float* dst0 = p.wpart + ((size_t)b * p.Hq + hq0) * hstride + (size_t)part * p.part_stride;
  const int ow = 2 + (p.v.qjl ? 2 * kHeadDim : kHeadDim);  // floats of one state (sketch part zero)
  if (cnt <= 0) {  // an empty part: the neutral state
    for (int i = tid; i < GH * ow; i += NT) dst0[(i / ow) * hstride + i % ow] = i % ow == 0 ? -INFINITY : 0.f;
    return;
  }
  const size_t pair = (size_t)b * p.Hkv + hk;
  const uint16_t* kw = p.wk + (pair * p.win_slots + t0) * kHeadDim;
  const uint16_t* vw = p.wv + (pair * p.win_slots + t0) * kHeadDim;
  for (int i = tid; i < GH * kHeadDim; i += NT) {
    const size_t qi = ((size_t)b * p.Hq + hq0 + i / kHeadDim) * kHeadDim + i % kHeadDim;
    qs[i] = (p.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[qi])
                    : reinterpret_cast<const float*>(p.q)[qi]) * p.logit_scale;
  }
  // keys: warp w, rows w TPW .. + TPW - 1 in batches of four (the next batch in flight while one
  // is used), lane l coordinates 4l .. 4l + 3
  auto load_k = [&](uint2 (&kr)[4], int r0) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
      kr[u] = r0 + u < cnt ? __ldcg(reinterpret_cast<const uint2*>(kw + (size_t)(r0 + u) * kHeadDim) + lane)
                           : make_uint2(0u, 0u);
  };
  uint2 kc[4], kn[4] = {};
  load_k(kc, warp * TPW);
  __syncthreads();  // the query
  // logits: per head, each lane's partial dot products of a batch's four rows, summed over the warp
  // by a reduce-scatter (3 shuffles leave row (lane >> 3) & 3 on a group of 8 lanes) and an
  // all-reduce within the group (3 more)
#pragma unroll 1
  for (int r0 = warp * TPW; r0 < (warp + 1) * TPW; r0 += 4) {
    if (r0 + 4 < (warp + 1) * TPW) load_k(kn, r0 + 4);
    float2 kf[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      kf[u][0] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kc[u].x));
      kf[u][1] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kc[u].y));
    }
#pragma unroll 1
    for (int h = 0; h < GH; ++h) {
      const float4 q4 = *reinterpret_cast<const float4*>(qs + h * kHeadDim + 4 * lane);
      float sv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        sv[u] = fmaf(kf[u][1].y, q4.w, fmaf(kf[u][1].x, q4.z, fmaf(kf[u][0].y, q4.y, kf[u][0].x * q4.x)));
      const bool up16 = (lane & 16) != 0, up8 = (lane & 8) != 0;
      sv[0] = (up16 ? sv[2] : sv[0]) + __shfl_xor_sync(0xffffffffu, up16 ? sv[0] : sv[2], 16);
      sv[1] = (up16 ? sv[3] : sv[1]) + __shfl_xor_sync(0xffffffffu, up16 ? sv[1] : sv[3], 16);
      sv[0] = (up8 ? sv[1] : sv[0]) + __shfl_xor_sync(0xffffffffu, up8 ? sv[0] : sv[1], 8);
#pragma unroll
      for (int off = 4; off > 0; off >>= 1) sv[0] += __shfl_xor_sync(0xffffffffu, sv[0], off);
      const int r = r0 + ((lane >> 3) & 3);
      if ((lane & 7) == 0) lg[h * kWinPart + r] = r < cnt ? sv[0] : -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) kc[u] = kn[u];
  }
  // values: thread (c2, tg) rows tg TPG .. + TPG - 1, coordinates 2 c2, 2 c2 + 1; the first batch
  // of eight is requested before the softmax
  const int c2 = tid & 63, tg = tid >> 6;
  auto load_v = [&](uint32_t (&vr)[8], int r0) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
      vr[u] = r0 + u < cnt ? __ldcg(reinterpret_cast<const unsigned int*>(vw + (size_t)(r0 + u) * kHeadDim) + c2) : 0u;
  };
  uint32_t vc[8], vn[8] = {};
  load_v(vc, tg * TPG);
  __syncthreads();
  // per head: max, weights 2^(l - m) in place, their sum (cnt >= 1, so the max is finite)
  for (int h = warp; h < GH; h += NW) {
    const float a = lg[h * kWinPart + lane], c = lg[h * kWinPart + 32 + lane];
    float mx = fmaxf(a, c);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float wa = exp2f(a - mx), wc = exp2f(c - mx);
    lg[h * kWinPart + lane] = wa;
    lg[h * kWinPart + 32 + lane] = wc;
    float sum = wa + wc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) {
      stat[2 * h] = mx;
      stat[2 * h + 1] = sum;
    }
  }
  __syncthreads();
  // o = sum_i w_i v_i: rows past cnt have weight 0 and zero values
  float acc[GH][2];
#pragma unroll
  for (int h = 0; h < GH; ++h) acc[h][0] = acc[h][1] = 0.f;
#pragma unroll 1
  for (int r0 = tg * TPG; r0 < (tg + 1) * TPG; r0 += 8) {
    if (r0 + 8 < (tg + 1) * TPG) load_v(vn, r0 + 8);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vc[u]));
#pragma unroll
      for (int h = 0; h < GH; ++h) {
        const float w = lg[h * kWinPart + r0 + u];
        acc[h][0] = fmaf(w, v.x, acc[h][0]);
        acc[h][1] = fmaf(w, v.y, acc[h][1]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) vc[u] = vn[u];
  }
#pragma unroll
  for (int h = 0; h < GH; ++h)
    *reinterpret_cast<float2*>(red + (tg * GH + h) * kHeadDim + 2 * c2) = make_float2(acc[h][0], acc[h][1]);
  __syncthreads();
  // sum the row groups; rotated caches take the signs (D o) here, then H / sqrt(d) below
  const float* sg = p.signs + hk * p.signs_stride;
  for (int i = tid; i < GH * kHeadDim; i += NT) {
    float o = 0.f;
#pragma unroll
    for (int g = 0; g < NG; ++g) o += red[g * GH * kHeadDim + i];
    red[i] = p.win_kivi ? o : o * sg[i % kHeadDim];
  }
  __syncthreads();
  // warp h: lane l holds coordinates 32k + l; butterflies over index bits 0..4 by shuffles, 5..6 in
  // registers (a KIVI cache is not rotated: the state stays in the original domain)
  for (int h = warp; h < GH; h += NW) {
    float* dst = dst0 + h * hstride;
    float u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = red[h * kHeadDim + 32 * k + lane];
    if (!p.win_kivi) {
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
      constexpr float kInvSqrtD = 0.08838834764831845f;  // 1/sqrt(128)
      u[0] = (a0 + a2) * kInvSqrtD;
      u[2] = (a0 - a2) * kInvSqrtD;
      u[1] = (a1 + a3) * kInvSqrtD;
      u[3] = (a1 - a3) * kInvSqrtD;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[2 + 32 * k + lane] = u[k];
    if (p.v.qjl)
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[2 + kHeadDim + 32 * k + lane] = 0.f;
    if (lane == 0) {
      dst[0] = stat[2 * h];
      dst[1] = stat[2 * h + 1];
    }
  }
}

}  // namespace kvq
