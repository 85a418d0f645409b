// KIVI-style appends ("TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers:
// TurboQuant and OSCAR": KIVI quantizes keys per channel -- keys have outlier channels that stay
// fixed across tokens -- and values per token). With b-bit asymmetric integers, for a group x:
//   z = min x, s = (max x - min x) / (2^b - 1), both rounded once to fp16 (saturating),
//   code = rint((x - z) / s) clipped to [0, 2^b - 1] (fp32 subtraction and IEEE division, ties to
//   even; s = 0 gives code 0); the estimate is z + s code.
// Keys take one (s, z) per channel over a group of 128 consecutive tokens, values one per token. A
// key group is coded once it is complete; until then its tokens stay in the cache's bf16 window (the
// incomplete last group), keys and values alike.
//
// kivi_groups: one block per (sequence, kv-head, group) an append completes. The group's 128 x 128
// keys, then its values, are staged in shared memory as fp32 (from the bf16 window for tokens stored
// before the call, from the input for the call's own); thread j takes key channel j (statistics and
// 128 codes, written as whole bytes of the octet-ordered planes: byte j-of-word holds one channel of
// 8 tokens), then thread t takes value token t (statistics and 128 codes as byte-lane-ordered
// planes). The four K and four V tiles of the group and its 512 bytes of key statistics are stored
// with 16-byte stores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kGroup = 128;   // tokens per key group (four tiles)
constexpr int kKiviThreads = 128;
constexpr int kXsStride = kGroup + 1;  // padded rows: column and row walks are both conflict-free

__device__ __forceinline__ float load_f(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}

__device__ __forceinline__ __half f16_sat(float x) { return __float2half_rn(fminf(fmaxf(x, -65504.f), 65504.f)); }

__device__ __forceinline__ int kivi_code(float x, float s, float z, int levels) {
  if (!(s > 0.f)) return 0;
  const float q = rintf(__fdiv_rn(x - z, s));
  return (int)fminf(fmaxf(q, 0.f), (float)(levels - 1));
}

__global__ void __launch_bounds__(kKiviThreads) kivi_groups(const __grid_constant__ QuantizeParams p, int max_groups) {
  extern __shared__ __align__(16) unsigned char ks_smem[];
  float* xs = reinterpret_cast<float*>(ks_smem);                          // [128 tokens][129]
  unsigned char* ktiles = ks_smem + sizeof(float) * kGroup * kXsStride;   // [4][k tile bytes]
  const SideLayout& KL = p.side[0];
  const SideLayout& VL = p.side[1];
  unsigned char* vtiles = ktiles + 4 * KL.tile_bytes;                     // [4][v tile bytes]
  __shared__ __align__(16) __half kstat[2][kHeadDim];
  const int tid = threadIdx.x;
  const int levels = 1 << KL.bits;
  const long total = (long)p.n_seq * p.heads * max_groups;
  for (long gidx = blockIdx.x; gidx < total; gidx += gridDim.x) {
    const int s = (int)(gidx / ((long)p.heads * max_groups));
    const int h = (int)((gidx / max_groups) % p.heads);
    const int gi = (int)(gidx % max_groups);
    const int T0 = p.total0[s], T1 = T0 + p.n_new;
    const int group = T0 / kGroup + gi;
    if (group >= T1 / kGroup) continue;  // the same for the whole block
    const int seq = p.seq[s], t_base = group * kGroup;
    const size_t pairidx = (size_t)seq * p.heads + h;
    for (int side = 0; side < 2; ++side) {
      // stage the group's vectors of this side: window rows below T0, input rows from T0 on
      for (int idx = tid; idx < kGroup * kHeadDim; idx += kKiviThreads) {
        const int t = idx / kHeadDim, j = idx % kHeadDim, pos = t_base + t;
        float x;
        if (pos < T0)
          x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.ring[side])[(pairidx * p.win_slots + pos % kGroup) * kHeadDim + j]);
        else
          x = load_f(p.src[side], (((size_t)s * p.heads + h) * p.n_new + (pos - T0)) * kHeadDim + j, p.bf16);
        xs[t * kXsStride + j] = x;
      }
      __syncthreads();
      if (side == 0) {
        // key channel j = tid: statistics over the group's tokens, then one byte per octet and plane
        const int j = tid;
        float lo = INFINITY, hi = -INFINITY;
        for (int t = 0; t < kGroup; ++t) {
          const float x = xs[t * kXsStride + j];
          lo = fminf(lo, x);
          hi = fmaxf(hi, x);
        }
        const __half s16 = f16_sat(__fdiv_rn(hi - lo, (float)(levels - 1))), z16 = f16_sat(lo);
        kstat[0][j] = s16;
        kstat[1][j] = z16;
        const float sf = __half2float(s16), zf = __half2float(z16);
        // octet order: word x = 8 t' + 2 m + hh, byte i is coordinate 32 m + 16 hh + 4 t' + i
        const int m = j >> 5, hh = (j >> 4) & 1, tq = (j >> 2) & 3, ib = j & 3;
        const int word = 8 * tq + 2 * m + hh;
        for (int o = 0; o < kGroup / 8; ++o) {  // 16 octets: tile o / 4, octet o % 4
          uint32_t bytes[3] = {0u, 0u, 0u};
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int c = kivi_code(xs[(8 * o + jj) * kXsStride + j], sf, zf, levels);
#pragma unroll
            for (int pl = 0; pl < 3; ++pl) bytes[pl] |= (uint32_t)((c >> pl) & 1) << jj;
          }
          unsigned char* tb = ktiles + (o >> 2) * KL.tile_bytes;
          for (int pl = 0; pl < KL.bits; ++pl)
            tb[KL.off_planes + pl * (kTile * 16) + (o & 3) * 128 + 4 * word + ib] = (unsigned char)bytes[pl];
        }
        if (tid < 32)  // the key tiles' norm slots are unused by KIVI caches: zero
          for (int q = 0; q < 4; ++q) reinterpret_cast<uint16_t*>(ktiles + q * KL.tile_bytes + KL.off_norm)[tid] = 0;
      } else {
        // value token t = tid: statistics over its channels, then its 16 bytes of every plane
        const int t = tid;
        float lo = INFINITY, hi = -INFINITY;
        for (int j = 0; j < kHeadDim; ++j) {
          const float x = xs[t * kXsStride + j];
          lo = fminf(lo, x);
          hi = fmaxf(hi, x);
        }
        const __half s16 = f16_sat(__fdiv_rn(hi - lo, (float)(levels - 1))), z16 = f16_sat(lo);
        const float sf = __half2float(s16), zf = __half2float(z16);
        unsigned char* tb = vtiles + (t >> 5) * VL.tile_bytes;
        const int slot = t & 31;
        for (int k = 0; k < kHeadDim / 8; ++k) {  // byte lane k: coordinates 8k .. 8k + 7
          uint32_t bytes[3] = {0u, 0u, 0u};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = kivi_code(xs[t * kXsStride + 8 * k + i], sf, zf, levels);
#pragma unroll
            for (int pl = 0; pl < 3; ++pl) bytes[pl] |= (uint32_t)((c >> pl) & 1) << i;
          }
          for (int pl = 0; pl < VL.bits; ++pl) tb[VL.off_planes + pl * (kTile * 16) + k * kTile + slot] = (unsigned char)bytes[pl];
        }
        *reinterpret_cast<__half*>(tb + VL.off_norm + 2 * slot) = s16;
        *reinterpret_cast<__half*>(tb + VL.off_gamma + 2 * slot) = z16;
      }
      __syncthreads();
    }
    // store the group: four K tiles, four V tiles, the key statistics
    char* kdst = p.region[0] + (pairidx * p.tiles_per_seq + 4 * group) * (size_t)KL.tile_bytes;
    char* vdst = p.region[1] + (pairidx * p.tiles_per_seq + 4 * group) * (size_t)VL.tile_bytes;
    for (int c = tid; c < 4 * KL.tile_bytes / 16; c += kKiviThreads)
      reinterpret_cast<uint4*>(kdst)[c] = reinterpret_cast<const uint4*>(ktiles)[c];
    for (int c = tid; c < 4 * VL.tile_bytes / 16; c += kKiviThreads)
      reinterpret_cast<uint4*>(vdst)[c] = reinterpret_cast<const uint4*>(vtiles)[c];
    char* sdst = p.kstats + (pairidx * p.groups_per_seq + group) * (size_t)(4 * kHeadDim);
    if (tid < 32) reinterpret_cast<uint4*>(sdst)[tid] = reinterpret_cast<const uint4*>(&kstat[0][0])[tid];
    __syncthreads();  // the next group reuses the staging and tile buffers
  }
  // history lengths: complete groups only
  if (blockIdx.x == 0)
    for (int i = tid; i < p.n_seq; i += kKiviThreads) p.lens[p.seq[i]] = (p.total0[i] + p.n_new) / kGroup * kGroup;
}

}  // namespace

cudaError_t launch_kivi_groups(const QuantizeParams& p, int max_groups, cudaStream_t s) {
  const size_t smem = sizeof(float) * kGroup * kXsStride + 4 * (size_t)(p.side[0].tile_bytes + p.side[1].tile_bytes);
  cudaError_t e = cudaFuncSetAttribute(kivi_groups, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  long blocks = (long)p.n_seq * p.heads * max_groups;
  if (blocks > 148L * 4) blocks = 148L * 4;
  kivi_groups<<<(int)(blocks < 1 ? 1 : blocks), kKiviThreads, smem, s>>>(p, max_groups);
  return launched();
}

}  // namespace kvq

// ---------------------------------------------------------------------------------------------
// KIVI decode over the coded history (complete key groups), CUDA cores, one CTA per (sequence,
// kv-head, split), 32-token tiles. Per key group: q'_h = q_h * s_g * scale * log2(e) and
// c_h = <q_h, z_g> * scale * log2(e), so a token's logit is c_h + sum_j q'_hj code_tj. Per tile:
// thread (slot t, quarter qq) sums channels 32 qq .. 32 qq + 31 of token t (octet-order key bits),
// then thread j accumulates value coordinate j: o_hj += p_t (z_t + s_t code_tj), with the running
// maximum rescaled as the tiles go (online softmax, base 2). Partials (m, l, o) in the original domain.
// ---------------------------------------------------------------------------------------------
namespace kvq {
namespace {

__device__ __forceinline__ float exp2_d(float a, float b) { return (a == -INFINITY) ? 0.f : exp2f(a - b); }

template <int G>
__global__ void __launch_bounds__(kKiviThreads) decode_kivi(const __grid_constant__ DecodeParams p) {
  __shared__ float qsm[G][kHeadDim];
  __shared__ float qp[G][kHeadDim];
  __shared__ float cz[G];
  __shared__ __align__(16) unsigned char kt[2 * kTile * 16];        // the tile's two key planes
  __shared__ __align__(16) unsigned char vt[2 * kTile * 16 + 128];  // value planes, s, z
  __shared__ float part[4][G][kTile];
  __shared__ float pw[G][kTile];       // weights 2^(l - m) of the tile
  __shared__ float mstat[G][2];        // running max, rescale factor of this tile
  const SideLayout& KL = p.k;
  const SideLayout& VL = p.v;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int len = p.lens[b];
  const int t_begin = split * p.chunk, t_end = min(len, t_begin + p.chunk);
  const size_t pair = (size_t)b * p.Hkv + hk;
  for (int i = tid; i < G * kHeadDim; i += kKiviThreads) {
    const int h = i / kHeadDim, j = i % kHeadDim;
    qsm[h][j] = load_f(p.q, ((size_t)b * p.Hq + hk * G + h) * kHeadDim + j, p.bf16) * p.logit_scale;
  }
  float m_run[G], l_run[G], o[G];  // thread j = tid: coordinate j of every head
#pragma unroll
  for (int h = 0; h < G; ++h) { m_run[h] = -INFINITY; l_run[h] = 0.f; o[h] = 0.f; }
  int cur_group = -1;
  const int t_slot = tid & 31, qq = tid >> 5;
  for (int tile = t_begin / kTile; tile * kTile < t_end; ++tile) {
    const int group = tile / 4;
    __syncthreads();  // the previous tile's buffers are free
    if (group != cur_group) {
      cur_group = group;
      const __half* st = reinterpret_cast<const __half*>(p.kstats + (pair * p.groups_per_seq + group) * (size_t)(4 * kHeadDim));
      const float sj = __half2float(st[tid]), zj = __half2float(st[kHeadDim + tid]);
#pragma unroll
      for (int h = 0; h < G; ++h) qp[h][tid] = qsm[h][tid] * sj;
      // c_h = sum_j q_hj z_j: warp sums, then across the four warps
      float zz[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = qsm[h][tid] * zj;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        zz[h] = v;
      }
      __syncthreads();
      if ((tid & 31) == 0)
#pragma unroll
        for (int h = 0; h < G; ++h) part[qq][h][0] = zz[h];
      __syncthreads();
      if (tid < G) cz[tid] = part[0][tid][0] + part[1][tid][0] + part[2][tid][0] + part[3][tid][0];
    }
    const char* ktile = p.kreg + (pair * p.tiles_per_seq + tile) * (size_t)KL.tile_bytes;
    const char* vtile = p.vreg + (pair * p.tiles_per_seq + tile) * (size_t)VL.tile_bytes;
    if (tid < 2 * kTile * 16 / 16) reinterpret_cast<uint4*>(kt)[tid] = reinterpret_cast<const uint4*>(ktile + KL.off_planes)[tid];
    if (tid < (2 * kTile * 16 + 128) / 16) reinterpret_cast<uint4*>(vt)[tid] = reinterpret_cast<const uint4*>(vtile + VL.off_planes)[tid];
    __syncthreads();
    // ---- logits: token t_slot, channels 32 qq .. 32 qq + 31 (words 8 tq + 2 qq + hh, bytes i)
    {
      const int o8 = t_slot >> 3, jj = t_slot & 7;
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int tq = 0; tq < 4; ++tq) {
          const int x = 8 * tq + 2 * qq + hh;
          const uint32_t w0 = reinterpret_cast<const uint32_t*>(kt)[o8 * 32 + x];
          const uint32_t w1 = reinterpret_cast<const uint32_t*>(kt + kTile * 16)[o8 * 32 + x];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = 32 * qq + 16 * hh + 4 * tq + i;
            const float code = (float)(((w0 >> (8 * i + jj)) & 1u) | (((w1 >> (8 * i + jj)) & 1u) << 1));
#pragma unroll
            for (int h = 0; h < G; ++h) acc[h] = fmaf(qp[h][c], code, acc[h]);
          }
        }
#pragma unroll
      for (int h = 0; h < G; ++h) part[qq][h][t_slot] = acc[h];
    }
    __syncthreads();
    // per head: the tile's logits, new running maximum, weights
    for (int idx = tid; idx < G * kTile; idx += kKiviThreads) {
      const int h = idx / kTile, t = idx % kTile;
      const bool ok = tile * kTile + t < t_end;
      pw[h][t] = ok ? cz[h] + part[0][h][t] + part[1][h][t] + part[2][h][t] + part[3][h][t] : -INFINITY;
    }
    __syncthreads();
    if (tid < G) {
      float mx = m_run[tid];
      for (int t = 0; t < kTile; ++t) mx = fmaxf(mx, pw[tid][t]);
      mstat[tid][0] = mx;
      mstat[tid][1] = exp2_d(m_run[tid], mx);
    }
    __syncthreads();
    for (int idx = tid; idx < G * kTile; idx += kKiviThreads) {
      const int h = idx / kTile, t = idx % kTile;
      pw[h][t] = exp2_d(pw[h][t], mstat[h][0]);
    }
    __syncthreads();
    // ---- values: coordinate j = tid (byte lane j / 8, bit j % 8)
    const int lane_k = tid >> 3, bit = tid & 7;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float c = mstat[h][1];
      o[h] *= c;
      l_run[h] *= c;
      m_run[h] = mstat[h][0];
    }
    for (int t = 0; t < kTile; ++t) {
      const int code = ((vt[lane_k * kTile + t] >> bit) & 1) | (((vt[kTile * 16 + lane_k * kTile + t] >> bit) & 1) << 1);
      const float sv = __half2float(*reinterpret_cast<const __half*>(vt + VL.off_norm - VL.off_planes + 2 * t));
      const float zv = __half2float(*reinterpret_cast<const __half*>(vt + VL.off_gamma - VL.off_planes + 2 * t));
      const float est = fmaf(sv, (float)code, zv);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        o[h] = fmaf(pw[h][t], est, o[h]);
        l_run[h] += pw[h][t];
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float* dst = p.part + (((size_t)b * p.Hq + hk * G + h) * p.splits + split) * p.part_stride;
    dst[2 + tid] = o[h];
    if (tid == 0) {
      dst[0] = m_run[h];
      dst[1] = l_run[h];
    }
  }
}

}  // namespace

cudaError_t launch_decode_kivi(const DecodeParams& p, cudaStream_t s) {
  const dim3 grid(p.splits, p.Hkv, p.B);
  switch (p.group) {
    case 1: decode_kivi<1><<<grid, kKiviThreads, 0, s>>>(p); break;
    case 2: decode_kivi<2><<<grid, kKiviThreads, 0, s>>>(p); break;
    case 4: decode_kivi<4><<<grid, kKiviThreads, 0, s>>>(p); break;
    case 8: decode_kivi<8><<<grid, kKiviThreads, 0, s>>>(p); break;
    default: return cudaErrorNotSupported;
  }
  return launched();
}

}  // namespace kvq
