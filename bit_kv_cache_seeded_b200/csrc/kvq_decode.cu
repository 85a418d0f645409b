// Split-K decode attention over an LM / LM_QJL / SIGN1 packed cache, and the split reduce.
//
// For one (sequence b, kv-head, context chunk) a CTA computes, for the g query heads of the
// group ("TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and
// OSCAR" -- logits from the Lloyd-Max centroids plus the unbiased QJL correction):
//   q_r = R q = H D q / sqrt(d),  s_q = S q_r                       (prologue, per head)
//   l_t = scale (n_t / sqrt d) [ <q_r, c[code_t]> + sqrt(pi/2)/m gamma_t <s_q, z_t> ]
//   online softmax in fp32 (base-2 exponent, log2(e) folded into the scale)
//   o_r   += p_t (n_t / sqrt d) c[code_t]                            (value centroids)
//   acc_z += p_t (n_t / sqrt d) sqrt(pi/2)/m gamma_t z_t             (value sketch, if any)
// and writes the partial (m, l, o_r, acc_z). The reduce kernel merges the splits,
//   M = max m_i, l = sum 2^(m_i - M) l_i, o = sum 2^(m_i - M) o_i / l,
// folds the value sketch back with S^T acc_z, and undoes the rotation: out = D H o / sqrt(d).
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_tiles.cuh"

namespace kvq {
namespace {

__device__ __forceinline__ float load_q(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
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

// exp2 that maps -inf to 0 without producing NaN for (-inf) - (-inf).
__device__ __forceinline__ float exp2_diff(float a, float b) {
  return (a == -INFINITY) ? 0.f : exp2f(a - b);
}

constexpr int kWarps = 4;

// 32-bit word k (coordinates 32k..32k+31) of token slot t of a plane at byte offset `off`
// (token or byte-lane order: the caches this kernel decodes never hold octet order).
__device__ __forceinline__ uint32_t vword(const char* tile, const SideLayout& L, int off, int t, int k) {
  if (L.order == kOrderToken) return *reinterpret_cast<const uint32_t*>(tile + off + t * 16 + k * 4);
  uint32_t w = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) w |= (uint32_t)(uint8_t)tile[off + (4 * k + b) * kTile + t] << (8 * b);
  return w;
}

// Rotated query of one head into smem: q_s = H D q * coef (coef folds 1/sqrt(d) and scales).
__device__ void rotate_query(const void* q, size_t base, int bf16, const float* signs, float coef,
                             float* dst) {
  const int lane = threadIdx.x & 31;
  float u[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) u[k] = load_q(q, base + 32 * k + lane, bf16) * signs[32 * k + lane];
#pragma unroll
  for (int b = 0; b < 5; ++b) {
    const bool upper = (lane >> b) & 1;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float o = __shfl_xor_sync(0xffffffffu, u[k], 1 << b);
      u[k] = upper ? o - u[k] : u[k] + o;
    }
  }
  const float a0 = u[0] + u[1], a1 = u[0] - u[1], a2 = u[2] + u[3], a3 = u[2] - u[3];
  dst[lane] = (a0 + a2) * coef;
  dst[64 + lane] = (a0 - a2) * coef;
  dst[32 + lane] = (a1 + a3) * coef;
  dst[96 + lane] = (a1 - a3) * coef;
}

template <int G, int KB, bool KQ, int VB, bool VQ>
__global__ void __launch_bounds__(kWarps * 32)
decode_lm_simple(const __grid_constant__ DecodeParams p) {
  __shared__ float q_s[G][kHeadDim];   // rotated query * scale/sqrt(d) * log2(e) / sqrt(d)
  __shared__ float s_s[G][kHeadDim];   // sketched query * the same * sqrt(pi/2)/m
  __shared__ float mrg[kWarps][G][2 + 2 * kHeadDim];
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int len = p.lens[b];
  const int t_begin = split * p.chunk;
  const int t_end = min(len, t_begin + p.chunk);
  const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)

  // ---- prologue: rotated (and sketched) queries of the group
  // logit (base 2) = n_t * ( <q_s, c> + gamma_t <s_s, z> ),  q_s = R q * scale*log2e/sqrt(d)
  const float qcoef = inv_sqrt_d * p.logit_scale * inv_sqrt_d;
  for (int h = warp; h < G; h += kWarps)
    rotate_query(p.q, ((size_t)b * p.Hq + hk * G + h) * kHeadDim, p.bf16, p.signs + hk * p.signs_stride, qcoef, q_s[h]);
  __syncthreads();
  if (KQ) {
    const float kappa = 1.2533141373155003f / (float)p.k.m;  // sqrt(pi/2)/m
    for (int idx = threadIdx.x; idx < G * kHeadDim; idx += blockDim.x) {
      const int h = idx / kHeadDim, j = idx % kHeadDim;
      float acc = 0.f;
      for (int i = 0; i < kHeadDim; ++i) acc = fmaf(p.St[(size_t)i * p.k.m + j], q_s[h][i], acc);
      s_s[h][j] = acc * kappa;
    }
  }
  __syncthreads();

  float m_run[G], l_run[G], o[G][4], oz[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m_run[h] = -INFINITY;
    l_run[h] = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) { o[h][k] = 0.f; oz[h][k] = 0.f; }
  }
  const float vkappa = VQ ? 1.2533141373155003f / (float)p.v.m : 0.f;

  for (int tile = t_begin / kTile + warp; tile * kTile < t_end; tile += kWarps) {
    const int count = min(kTile, t_end - tile * kTile);
    const bool valid = lane < count;
    const long ti = tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk, tile, p.err);
    const char* kt = p.kreg + (size_t)ti * p.k.tile_bytes;
    const char* vt = p.vreg + (size_t)ti * p.v.tile_bytes;

    // ---- logits: lane = token
    float logit[G];
    {
      uint4 pl[KB];
#pragma unroll
      for (int pp = 0; pp < KB; ++pp)
        pl[pp] = *reinterpret_cast<const uint4*>(kt + p.k.off_planes + pp * (kTile * 16) + lane * 16);
      uint4 zz = make_uint4(0, 0, 0, 0);
      float gam = 0.f;
      if (KQ) {
        zz = *reinterpret_cast<const uint4*>(kt + p.k.off_sketch + lane * 16);
        gam = __half2float(*reinterpret_cast<const __half*>(kt + p.k.off_gamma + lane * 2));
      }
      const float nk = __half2float(*reinterpret_cast<const __half*>(kt + p.k.off_norm + lane * 2));
      float dot[G], dz[G];
#pragma unroll
      for (int h = 0; h < G; ++h) { dot[h] = 0.f; dz[h] = 0.f; }
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t words[KB];
#pragma unroll
        for (int pp = 0; pp < KB; ++pp)
          words[pp] = (w == 0) ? pl[pp].x : (w == 1) ? pl[pp].y : (w == 2) ? pl[pp].z : pl[pp].w;
        const uint32_t zword = (w == 0) ? zz.x : (w == 1) ? zz.y : (w == 2) ? zz.z : zz.w;
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          int code = 0;
#pragma unroll
          for (int pp = 0; pp < KB; ++pp) code |= ((words[pp] >> i) & 1) << pp;
          const float c = p.k.cent[code];
          const int j = 32 * w + i;
#pragma unroll
          for (int h = 0; h < G; ++h) dot[h] = fmaf(q_s[h][j], c, dot[h]);
          if (KQ) {
            const float zs = ((zword >> i) & 1) ? 1.f : -1.f;
#pragma unroll
            for (int h = 0; h < G; ++h) dz[h] = fmaf(s_s[h][j], zs, dz[h]);
          }
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) logit[h] = valid ? nk * (dot[h] + (KQ ? gam * dz[h] : 0.f)) : -INFINITY;
    }

    // ---- online softmax (per warp, per head)
    float pw[G], pz[G];
    const float nv = valid ? __half2float(*reinterpret_cast<const __half*>(vt + p.v.off_norm + lane * 2)) * inv_sqrt_d : 0.f;
    const float gv = (VQ && valid) ? __half2float(*reinterpret_cast<const __half*>(vt + p.v.off_gamma + lane * 2)) * vkappa : 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float m_new = fmaxf(m_run[h], warp_max(logit[h]));
      const float corr = exp2_diff(m_run[h], m_new);
      const float pr = exp2_diff(logit[h], m_new);
      l_run[h] = l_run[h] * corr + warp_sum(pr);
      m_run[h] = m_new;
#pragma unroll
      for (int k = 0; k < 4; ++k) { o[h][k] *= corr; oz[h][k] *= corr; }
      pw[h] = pr * nv;
      pz[h] = pw[h] * gv;
    }

    // ---- values: lane = coordinate (32k + lane), loop over the tile's tokens
    for (int t = 0; t < count; ++t) {
      uint32_t vw[VB][4];
#pragma unroll
      for (int pp = 0; pp < VB; ++pp)
#pragma unroll
        for (int k = 0; k < 4; ++k) vw[pp][k] = vword(vt, p.v, p.v.off_planes + pp * (kTile * 16), t, k);
      float c[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int code = 0;
#pragma unroll
        for (int pp = 0; pp < VB; ++pp) code |= ((vw[pp][k] >> lane) & 1) << pp;
        c[k] = p.v.cent[code];
      }
      float zs[4] = {0.f, 0.f, 0.f, 0.f};
      if (VQ) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          zs[k] = ((vword(vt, p.v, p.v.off_sketch, t, k) >> lane) & 1) ? 1.f : -1.f;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pt = __shfl_sync(0xffffffffu, pw[h], t);
#pragma unroll
        for (int k = 0; k < 4; ++k) o[h][k] = fmaf(pt, c[k], o[h][k]);
        if (VQ) {
          const float ptz = __shfl_sync(0xffffffffu, pz[h], t);
#pragma unroll
          for (int k = 0; k < 4; ++k) oz[h][k] = fmaf(ptz, zs[k], oz[h][k]);
        }
      }
    }
  }

  // ---- merge the CTA's warps and write the split partial
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (lane == 0) { mrg[warp][h][0] = m_run[h]; mrg[warp][h][1] = l_run[h]; }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      mrg[warp][h][2 + 32 * k + lane] = o[h][k];
      mrg[warp][h][2 + kHeadDim + 32 * k + lane] = oz[h][k];
    }
  }
  __syncthreads();
  const int width = 2 + (VQ ? 2 : 1) * kHeadDim;
  for (int idx = threadIdx.x; idx < G * width; idx += blockDim.x) {
    const int h = idx / width, e = idx % width;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mrg[w][h][0]);
    float v = 0.f;
    if (e == 0) {
      v = M;
    } else {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += exp2_diff(mrg[w][h][0], M) * mrg[w][h][e];
    }
    float* dst = p.part + (((size_t)b * p.Hq + hk * G + h) * p.splits + split) * p.part_stride;
    dst[e] = v;
  }
}

// One block per (sequence, kv-head), 128 threads per query head of the group. Merge: thread
// (h, i) merges head h's split partials at coordinate i (the loads of 8 splits issued together,
// one memory latency per 8 splits). Value sketch fold-back, o_r += S^T acc_z, with S staged in
// shared memory by cp.async while the partials are merged: thread (q, i) sums the rows j of
// quarter q (of G) for all G heads at once, so each staged S element is read once; the G partial
// sums of a head meet in shared memory. Warp h then undoes the rotation of head h
// (out = D H o_r / sqrt(d)) with shuffles and writes it out.
template <int G>
__global__ void __launch_bounds__(G * kHeadDim)
reduce_lm(const __grid_constant__ DecodeParams p, int vq) {
  constexpr int kSplitBatch = 8;
  constexpr int kRows = kHeadDim / G;                 // sketch rows per thread in the fold-back
  extern __shared__ __align__(16) float rs[];
  float* S_s = rs;                                   // [m][d] when vq
  float* az = rs + (vq ? p.v.m * kHeadDim : 0);      // [m][G] merged sketch accumulators
  float* xs = az + G * kHeadDim;                     // [G][d] rotated-domain outputs
  float* red = xs + G * kHeadDim;                    // [G quarters][G heads][d] fold-back partials
  const int hk = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int h = tid / kHeadDim, i = tid % kHeadDim;
  const int lane = tid & 31, warp = tid >> 5;
  grid_dep_launch();  // a following fused step's first kernel may start its setup now
  if (vq) {
    for (int c = tid; c < p.v.m * kHeadDim / 4; c += G * kHeadDim) cp_async16(S_s + 4 * c, p.S + 4 * c);
    cp_async_commit();
  }
  float sg[4];  // the output rotation's signs and scale (warps 0..G-1), fetched while waiting
#pragma unroll
  for (int k = 0; k < 4; ++k) sg[k] = warp < G ? p.signs[hk * p.signs_stride + 32 * k + lane] * 0.08838834764831845f : 0.f;
  // Launched as a programmatic dependent of the decode kernel: S is staged above while that
  // grid finishes; its partials are read only after this wait.
  grid_dep_wait();
  float M = -INFINITY, L = 0.f, o = 0.f, oz = 0.f;
  // fold n consecutive states [n][part_stride] into (M, L, o, oz), kSplitBatch loads in flight
  auto merge = [&](const float* part, int n) {
    for (int s0 = 0; s0 < n; s0 += kSplitBatch) {
      float mv[kSplitBatch], lv[kSplitBatch], ov[kSplitBatch], zv[kSplitBatch];
#pragma unroll
      for (int k = 0; k < kSplitBatch; ++k) {
        const bool in = s0 + k < n;
        const float* ps = part + (size_t)(in ? s0 + k : 0) * p.part_stride;
        mv[k] = in ? __ldcg(ps) : -INFINITY;
        lv[k] = in ? __ldcg(ps + 1) : 0.f;
        ov[k] = in ? __ldcg(ps + 2 + i) : 0.f;
        zv[k] = (in && vq) ? __ldcg(ps + 2 + kHeadDim + i) : 0.f;
      }
      float mn = M;
#pragma unroll
      for (int k = 0; k < kSplitBatch; ++k) mn = fmaxf(mn, mv[k]);
      const float c = exp2_diff(M, mn);
      L *= c; o *= c; oz *= c;
#pragma unroll
      for (int k = 0; k < kSplitBatch; ++k) {
        const float w = exp2_diff(mv[k], mn);
        L = fmaf(w, lv[k], L);
        o = fmaf(w, ov[k], o);
        oz = fmaf(w, zv[k], oz);
      }
      M = mn;
    }
  };
  merge(p.part + ((size_t)b * p.Hq + hk * G + h) * (size_t)p.splits * p.part_stride, p.splits);
  // the mixed-precision window's parts: more terms of the same softmax
  if (p.wpart) merge(p.wpart + ((size_t)b * p.Hq + hk * G + h) * (size_t)p.win_parts * p.part_stride, p.win_parts);
  // the normalisation by L, unless the call asks for the merged softmax state (m, l, unnormalised
  // o), whose Sᵀ fold and inverse rotation are linear and apply the same way
  const float inv = p.pout ? 1.f : (L > 0.f) ? 1.f / L : 0.f;
  o *= inv;
  if (vq) {
    az[i * G + h] = oz * inv;
    cp_async_wait<0>();
    __syncthreads();
    const int q = h;  // this thread's quarter of the sketch rows
    float acc[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) acc[hh] = 0.f;
#pragma unroll 8
    for (int j = q * kRows; j < (q + 1) * kRows; ++j) {
      const float sv = S_s[j * kHeadDim + i];
      if (G >= 4) {
#pragma unroll
        for (int h4 = 0; h4 < G; h4 += 4) {
          const float4 a = *reinterpret_cast<const float4*>(az + j * G + h4);
          acc[h4] = fmaf(sv, a.x, acc[h4]);
          acc[h4 + 1] = fmaf(sv, a.y, acc[h4 + 1]);
          acc[h4 + 2] = fmaf(sv, a.z, acc[h4 + 2]);
          acc[h4 + 3] = fmaf(sv, a.w, acc[h4 + 3]);
        }
      } else {
#pragma unroll
        for (int hh = 0; hh < G; ++hh) acc[hh] = fmaf(sv, az[j * G + hh], acc[hh]);
      }
    }
#pragma unroll
    for (int hh = 0; hh < G; ++hh) red[(q * G + hh) * kHeadDim + i] = acc[hh];
    __syncthreads();
#pragma unroll
    for (int qq = 0; qq < G; ++qq) o += red[(qq * G + h) * kHeadDim + i];
  }
  xs[h * kHeadDim + i] = o;
  __syncthreads();
  // lane l of warp h holds coordinates 32k + l; butterflies over index bits 0..4 by shuffles,
  // bits 5..6 in registers. KIVI caches are not rotated: the output is o itself.
  if (p.win_kivi && warp < G) {
    const int hh = warp;
    float* dst = p.pout ? p.pout + ((size_t)b * p.Hq + hk * G + hh) * (2 + kHeadDim) + 2
                        : p.out + ((size_t)b * p.Hq + hk * G + hh) * kHeadDim;
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[32 * k + lane] = xs[hh * kHeadDim + 32 * k + lane];
  } else if (warp < G) {
    const int hh = warp;
    float u[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = xs[hh * kHeadDim + 32 * k + lane];
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
    float* dst = p.pout ? p.pout + ((size_t)b * p.Hq + hk * G + hh) * (2 + kHeadDim) + 2
                        : p.out + ((size_t)b * p.Hq + hk * G + hh) * kHeadDim;
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[32 * k + lane] = u[k] * sg[k];
  }
  if (p.pout && i == 0) {  // the head's running maximum (log2 units) and sum of weights
    float* st = p.pout + ((size_t)b * p.Hq + hk * G + h) * (2 + kHeadDim);
    st[0] = M;
    st[1] = L;
  }
}

template <int G>
cudaError_t dispatch_modes(const DecodeParams& p, dim3 grid, cudaStream_t s) {
  const int kb = p.k.bits, vb = p.v.bits;
  const bool kq = p.k.qjl, vq = p.v.qjl;
#define KVQ_CASE(KB, KQ, VB, VQ)                                              \
  if (kb == KB && kq == KQ && vb == VB && vq == VQ) {                         \
    decode_lm_simple<G, KB, KQ, VB, VQ><<<grid, kWarps * 32, 0, s>>>(p);      \
    return launched();                                                        \
  }
  KVQ_CASE(2, true, 2, true)
  KVQ_CASE(3, true, 3, false)
  KVQ_CASE(1, false, 1, false)
  KVQ_CASE(2, true, 2, false)
  KVQ_CASE(3, true, 3, true)
  KVQ_CASE(2, false, 2, false)
  KVQ_CASE(3, false, 3, false)
  KVQ_CASE(1, true, 1, false)
  KVQ_CASE(1, true, 1, true)
#undef KVQ_CASE
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_decode_lm(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  if (p.use_tc) {
    if (!tc_decode_supported(p)) return cudaErrorNotSupported;
    return p.use_tc == 2 ? launch_decode_lm_ws(p, s, ev_mid, qp) : launch_decode_lm_tc(p, s, ev_mid, qp);
  }
  if (mma_decode_supported(p)) return launch_decode_lm_mma(p, s, ev_mid, qp);
  if (qp) return cudaErrorNotSupported;
  if (ev_mid && cudaEventRecord(ev_mid, s) != cudaSuccess) return cudaErrorUnknown;
  dim3 grid(p.splits, p.Hkv, p.B);
  switch (p.group) {
    case 1: return dispatch_modes<1>(p, grid, s);
    case 2: return dispatch_modes<2>(p, grid, s);
    case 4: return dispatch_modes<4>(p, grid, s);
    case 8: return dispatch_modes<8>(p, grid, s);
    default: return cudaErrorNotSupported;
  }
}

template <int G>
cudaError_t launch_reduce_g(const DecodeParams& p, cudaStream_t s) {
  const size_t smem = sizeof(float) * ((p.v.qjl ? (size_t)p.v.m * kHeadDim : 0) + 2 * G * kHeadDim +
                                      (size_t)G * G * kHeadDim);
  cudaError_t e = cudaFuncSetAttribute(reduce_lm<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.Hkv, p.B);
  cfg.blockDim = dim3(G * kHeadDim);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, reduce_lm<G>, p, (int)p.v.qjl);
  if (e != cudaSuccess) return e;
  return launched();
}

cudaError_t launch_reduce_lm(const DecodeParams& p, cudaStream_t s) {
  switch (p.group) {
    case 1: return launch_reduce_g<1>(p, s);
    case 2: return launch_reduce_g<2>(p, s);
    case 4: return launch_reduce_g<4>(p, s);
    case 8: return launch_reduce_g<8>(p, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kvq
