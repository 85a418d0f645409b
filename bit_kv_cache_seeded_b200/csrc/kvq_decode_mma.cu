// Tensor-core split-K decode attention for LM / LM_QJL / SIGN1 caches (up to 4 query heads per
// CTA; a query group of 8 runs as two pieces of 4 heads).
//
// Same computation as the CUDA-core kernel in kvq_decode.cu ("TurboQuant vs OSCAR vs
// EpiCache", section "Quantization frontiers: TurboQuant and OSCAR": logits from the
// Lloyd-Max centroids plus the unbiased QJL correction, softmax, values dequantised on the fly),
// arranged as exact int8 tensor-core contractions (mma.sync m16n8k32 s8 -> s32) over the packed
// bit-planes:
//
//   * Walsh expansion of the code table. The Lloyd-Max table is odd, so with B_i = 2 b_i - 1:
//       1 bit : c = a0 B0;   2 bits: c = a0 B0 + a1 B1
//       3 bits: c = a0 B0 + a1 B1 + a2 B2 + a3 B0B1B2,   B0B1B2 = 2 (b0^b1^b2) - 1
//     so <q, c[code]> = sum_P 2 a_P <q, b_P> - (sum_P a_P) sum_j q_j over 0/1 "Walsh planes".
//   * Logits: A = key bits [16 tokens x 32 coordinates] from the octet-ordered key tile, where a
//     byte holds one coordinate of 8 consecutive tokens: w & (0x01010101 << g) keeps token g of
//     the octet in every byte, the int8 value 2^g (g < 7) or -128 (g = 7), one LOP3 per 4 operand
//     bytes and a fixed power of two per row. B = the query term 2 a_P q~_j quantised to a
//     16-bit integer (2 signed 8-bit digits, one column each).
//   * Values: A = value bits [16 coordinates x 32 tokens] read from the byte-lane-major value
//     tile, where 4 tokens of one byte-lane are one 32-bit word: w & (0x01010101 << p) gives the
//     int8 value 2^p (p < 7) or -128 (p = 7) per byte, i.e. a fixed power of two per row. B = the
//     softmax weights p_t n_t / sqrt(d) (times sqrt(pi/2)/m gamma_t for the value sketch) as a
//     23-bit integer (3 unsigned byte digits), each kind scaled by a power of two to its own
//     chunk maximum.
//   * Two passes over a CTA's chunk (at most kChunkMax tokens): pass 1 computes every logit into
//     shared memory and the chunk's maxima; pass 2 streams the value tiles with the weights
//     2^(l - M) fixed, so the int32 accumulators are exact and never rescaled.
//
// CTA: 4 warps. Pass 1: 64 tokens (two cache tiles) per iteration, warp w owns tokens
// 16w..16w+15. Pass 2: 64 tokens per iteration, warp w owns bit positions 2w, 2w+1 of every value
// Walsh plane. Both passes stream whole tile pairs through 4 shared-memory stages with bulk
// (TMA 1-D) copies completing on mbarriers; the value tiles of pass 2 are already in flight during
// the last iterations of pass 1. Every wait is bounded: a wait that gives up sets bit 0 of the
// cache's status word. Partials (m, l, o_r, acc_z) are written in the format of the CUDA-core
// kernel; the same reduce kernel finishes.
#include <algorithm>
#include <type_traits>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_quantize_lm.cuh"
#include "kvq_lm_common.cuh"
#include "kvq_tiles.cuh"
#include "kvq_window.cuh"

namespace kvq {
namespace {

using namespace lmc;

constexpr int kWarpsM = 4;
constexpr int kThreadsM = kWarpsM * 32;
constexpr int kCtaTok = 64;
constexpr int kStagesM = 4;                          // bulk-copy stages (tile pairs in flight)
constexpr int kSmemPerSm = 233472;                   // shared memory per SM (228 KB)
constexpr int kSmemReserved = 1024 + 128;            // per CTA: the runtime's reserve + static arrays
constexpr int kPdStride = 96;                        // weight-digit row stride (bytes): 64 tokens + pad
constexpr int kNormBlock = 256;                      // staged value norms / gammas of two cache tiles
constexpr int kKeyChains = 2;                        // independent key accumulators (coordinate blocks m % 2)

// A int8, B uint8 (the value-phase weight digits are non-negative bytes).
__device__ __forceinline__ void mma_s8u8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte `k` of each of four words, packed into one word (k = 0..3).
template <int K>
__device__ __forceinline__ uint32_t pack_byte(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3) {
  const uint32_t a = __byte_perm(x0, x1, K | ((4 + K) << 4));
  const uint32_t b = __byte_perm(x2, x3, K | ((4 + K) << 4));
  return __byte_perm(a, b, 0x5410);
}

__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Bit p of every byte of w as the int8 value -128 (set) or 0 (clear).
template <int P>
__device__ __forceinline__ uint32_t bit_to_s8(uint32_t w) {
  return (P == 7) ? (w & 0x80808080u) : ((w * (1u << (7 - P))) & 0x80808080u);
}

// Warps of a decode CTA: 4, or 8 for a query group of 8 (one CTA per kv-head: warps w and w + 4
// take the same tokens for heads 0-3 and 4-7 in pass 1, and one value bit position each in pass 2).
template <int G> struct Warps { static constexpr int N = G > 4 ? 8 : 4; };

template <int G, int KB, bool KQ, int VB, bool VQ>
struct MmaCfg {
  static constexpr int NW = Warps<G>::N, NT = NW * 32;
  static constexpr int GW = G > 4 ? 4 : G;                // heads of one warp's logits
  static constexpr int KP = Walsh<KB>::P + (KQ ? 1 : 0);  // logit planes (sketch last)
  static constexpr int VP = Walsh<VB>::P + (VQ ? 1 : 0);  // value planes (sketch last)
  static constexpr int KNT = (2 * GW + 7) / 8;            // logit N-tiles: (head, 2 digits)
  static constexpr int VNT = (3 * G + 7) / 8;             // value N-tiles: (head, 3 digits), column 3h + d
  static constexpr int VNCOL = VNT * 8;
  static constexpr int PPW = 8 / NW;                      // value bit positions per warp
};

// Dynamic shared memory of one decode CTA: the staging ring, the chunk's logits, the two weight
// digit buffers and the reduction scratch.
size_t mma_smem_bytes(int group, const SideLayout& k, const SideLayout& v, int chunk, bool kivi) {
  const int nkind = v.qjl ? 2 : 1;
  const int vncol = ((3 * group + 7) / 8) * 8;
  const int nw = group > 4 ? 8 : 4;
  size_t s = (size_t)kStagesM * std::max(2 * k.tile_bytes + kNormBlock + (kivi ? kKiviStats : 0), 2 * v.tile_bytes);
  s += sizeof(float) * (size_t)group * (chunk + 8);
  s += 2 * (size_t)nkind * vncol * kPdStride;
  s += sizeof(float) * (nw * group + 2 * nw);
  if (kivi)  // query, the group's two-plane digit table, head constants
    s += sizeof(float) * (size_t)group * kHeadDim + 2 * (size_t)group * 2 * kHeadDim + sizeof(float) * 2 * group;
  return (s + 15) / 16 * 16;
}

// ------------------------------------------------------------------------------------------
// Prep kernel, once per (sequence, kv-head): the logit-phase B operand.
//   q~ = H D q * scale*log2(e)/d (rotated query),  s~ = sqrt(pi/2)/m * S q~ (sketched query)
//   centroid planes: v = 2 a_P q~_j;  sketch plane: v = 2 s~_j
//   q_int = rint(v * 32639 / vmax_h) (vmax over the centroid planes, separately for the sketch),
//   digits hi = floor((q_int + 128) / 256) in [-127, 127], lo = q_int - 256 hi in [-128, 128):
//   two full int8 digits, about 16 bits of the query term.
// Layout per pair: [KP][G][2 digits][128 fragment-ordered coordinates] bytes, then [G][4] f32:
// (s, C, sz, Cz) with s = vmax / (32639 * -128) (the one-hot bytes are -128), C = -(sum_P a_P)
// sum_j q~_j and Cz = -sum_j s~_j. Coordinates in natural order: the decode kernel's operand byte
// k of coordinate block m is coordinate 32m + k.
// ------------------------------------------------------------------------------------------
template <int G, int KB, bool KQ>
__device__ __forceinline__ void prep_block(const DecodeParams& p, int vk, int b) {
  constexpr int KP = Walsh<KB>::P + (KQ ? 1 : 0);
  constexpr int KWP = Walsh<KB>::P;
  __shared__ __align__(16) float qf[G][kHeadDim];
  __shared__ __align__(16) float sf[G][kHeadDim];
  __shared__ float hc[G][4];
  __shared__ float qscale[G][2];                 // 32639 / vmax: centroid planes, sketch
  __shared__ __align__(8) uint64_t st_bar;       // completes when S^T has landed
  extern __shared__ __align__(16) float st_s[];  // [128][m] transposed sketch matrix
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // piece `half` (of p.hsplit) of kv-head hk's query group: query heads h_first .. h_first + G - 1
  const int hk = vk / p.hsplit, half = vk % p.hsplit;
  const int h_first = hk * p.group + half * G;
  unsigned char* out = p.qprep + (((size_t)b * p.Hkv + hk) * p.hsplit + half) * p.qprep_stride;
  static_assert(G <= kWarpsM, "one query head per warp");
  const int h0 = warp;  // this warp's query head (h0 < G)
  if (KQ && tid == 0) {  // one bulk copy, landing while the queries are rotated
    const uint32_t bar = smem_addr(&st_bar);
    mbar_init(bar, 1);
    mbar_init_fence();
    constexpr uint32_t kQuarter = kHeadDim * kHeadDim / 4;  // floats in a quarter of S^T (16 KB)
    mbar_arrive_expect_tx(bar, 4u * kQuarter * 4u);
#pragma unroll
    for (int c = 0; c < 4; ++c) bulk_g2s(smem_addr(st_s + c * kQuarter), p.St + c * kQuarter, kQuarter * 4u, bar);
  }
  float u[4];
  // Launched as a programmatic dependent (fused decode step): the query may come from the
  // preceding kernel, so wait for it (the sketch matrix requested above is the cache's own).
  grid_dep_wait();
  if (h0 < G) {
    const size_t qb = ((size_t)b * p.Hq + h_first + h0) * kHeadDim;
#pragma unroll
    for (int k = 0; k < 4; ++k) u[k] = load_q(p.q, qb + 32 * k + lane, p.bf16) * p.signs[hk * p.signs_stride + 32 * k + lane];
  }
  const float qcoef = kInvSqrtD * p.logit_scale * kInvSqrtD;
  if (h0 < G) {
#pragma unroll
    for (int bb = 0; bb < 5; ++bb) {
      const bool upper = (lane >> bb) & 1;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float o = __shfl_xor_sync(0xffffffffu, u[k], 1 << bb);
        u[k] = upper ? o - u[k] : u[k] + o;
      }
    }
    const float a0 = u[0] + u[1], a1 = u[0] - u[1], a2 = u[2] + u[3], a3 = u[2] - u[3];
    qf[h0][lane] = (a0 + a2) * qcoef;
    qf[h0][64 + lane] = (a0 - a2) * qcoef;
    qf[h0][32 + lane] = (a1 + a3) * qcoef;
    qf[h0][96 + lane] = (a1 - a3) * qcoef;
  }
  __syncthreads();  // the rotated queries; the barrier below was initialised before this
  bool st_failed = false;
  if (KQ && !mbar_try(smem_addr(&st_bar), 0u) && !mbar_wait(smem_addr(&st_bar), 0u, p.wait_limit)) {
    st_failed = true;
    atomicOr(p.err, 1);
  }
  if (KQ) {
    const float kappa = kSqrtHalfPi / (float)p.k.m;
    const int j = tid;  // 128 threads, one sketch row each; two halves of the sum as separate chains
    float acc[2][G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[0][h] = acc[1][h] = 0.f;
#pragma unroll 2
    for (int i = 0; i < kHeadDim / 2; i += 4) {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        const int ii = i + hf * (kHeadDim / 2);
        const float s0 = st_s[ii * kHeadDim + j], s1 = st_s[(ii + 1) * kHeadDim + j];
        const float s2 = st_s[(ii + 2) * kHeadDim + j], s3 = st_s[(ii + 3) * kHeadDim + j];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float4 qv = *reinterpret_cast<const float4*>(&qf[h][ii]);
          acc[hf][h] = fmaf(s3, qv.w, fmaf(s2, qv.z, fmaf(s1, qv.y, fmaf(s0, qv.x, acc[hf][h]))));
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) sf[h][j] = (acc[0][h] + acc[1][h]) * kappa;
    __syncthreads();
  }
  float ka[4];
  walsh_coeffs(KB, p.k.cent, ka);
  for (int task = warp; task < 2 * G; task += kWarpsM) {  // (head, 0: centroid planes / 1: sketch)
    const int h = task >> 1, which = task & 1;
    float mx = 0.f, sum = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float v = which ? sf[h][32 * k + lane] : qf[h][32 * k + lane];
      mx = fmaxf(mx, fabsf(v));
      sum += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    float asum = 0.f, amax = 0.f;
#pragma unroll
    for (int P = 0; P < KWP; ++P) { asum += ka[P]; amax = fmaxf(amax, fabsf(ka[P])); }
    mx *= which ? 2.f : 2.f * amax;  // largest |v| over the planes
    if (lane == 0) {
      hc[h][2 * which] = mx > 0.f ? mx : 1.f;
      hc[h][2 * which + 1] = which ? -sum : -asum * sum;
      qscale[h][which] = (float)kQRange / (mx > 0.f ? mx : 1.f);
    }
  }
  __syncthreads();
  // four consecutive coordinates per step: their hi and lo digits are one 32-bit store each
  for (int idx = tid; idx < KP * G * (kHeadDim / 4); idx += kThreadsM) {
    const int P = idx / (G * (kHeadDim / 4)), h = (idx / (kHeadDim / 4)) % G, j0 = 4 * (idx % (kHeadDim / 4));
    const bool sk = KQ && P == KP - 1;
    float kaP = ka[0];
#pragma unroll
    for (int r = 1; r < 4; ++r)
      if (P == r) kaP = ka[r];
    const float4 src = sk ? *reinterpret_cast<const float4*>(&sf[h][j0]) : *reinterpret_cast<const float4*>(&qf[h][j0]);
    const float mul = (sk ? 2.f : 2.f * kaP);
    const float qs = qscale[h][sk ? 1 : 0];
    const float vv[4] = {src.x, src.y, src.z, src.w};
    uint32_t hw = 0u, lw = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int q = __float2int_rn((mul * vv[e]) * qs);
      const int hi = (q + 128) >> 8, lo = q - 256 * hi;
      hw |= (uint32_t)(hi & 0xFF) << (8 * e);
      lw |= (uint32_t)(lo & 0xFF) << (8 * e);
    }
    *reinterpret_cast<uint32_t*>(out + ((P * G + h) * 2 + 0) * 128 + j0) = hw;
    *reinterpret_cast<uint32_t*>(out + ((P * G + h) * 2 + 1) * 128 + j0) = lw;
  }
  __syncthreads();
  if (st_failed) mbar_wait(smem_addr(&st_bar), 0u, p.wait_limit);  // nothing may land after exit
  if (tid < 4 * G) {
    const int h = tid / 4, k = tid % 4;
    float v = hc[h][k];
    if (k == 0 || k == 2) v = v / ((float)kQRange * -128.f);  // integer sum -> query units
    reinterpret_cast<float*>(out + KP * G * 2 * 128)[tid] = v;
  }
}

template <int G, int KB, bool KQ>
__global__ void __launch_bounds__(kThreadsM) decode_lm_prep(const __grid_constant__ DecodeParams p) {
  grid_dep_launch();  // the decode kernel may be scheduled now; it waits before reading this output
  prep_block<G, KB, KQ>(p, blockIdx.x, blockIdx.y);
}

// Front kernel of a fused decode step (kvq_decode_step): blocks 0 .. 2 nq - 1 append the new
// token of every sequence (K side, then V side: qlm::quantize_lm_block), the remaining B x Hkv
// blocks compute the query prep. The two parts are independent, so they share one launch and
// overlap; the decode kernel, a programmatic dependent of this one, waits for all of it.
template <int G, int KB, bool KQ>
__global__ void __launch_bounds__(kThreadsM)
decode_front(const __grid_constant__ QuantizeParams qp, const __grid_constant__ DecodeParams p, int nq) {
  grid_dep_launch();
  const int blk = blockIdx.x;
  if (blk < 2 * nq) {
    qlm::quantize_lm_block(qp, blk / nq, blk % nq, nq);
  } else {
    const int r = blk - 2 * nq;
    prep_block<G, KB, KQ>(p, r % (p.Hkv * p.hsplit), r / (p.Hkv * p.hsplit));
  }
}

// ------------------------------------------------------------------------------------------
// Decode kernel (two passes over the CTA's chunk).
// ------------------------------------------------------------------------------------------
template <int G, int KB, bool KQ, int VB, bool VQ, bool KV>
__global__ void __launch_bounds__(Warps<G>::N * 32, 16 / Warps<G>::N)
decode_lm_mma(const __grid_constant__ DecodeParams p) {
  using C = MmaCfg<G, KB, KQ, VB, VQ>;
  constexpr int KP = C::KP, VP = C::VP, KNT = C::KNT, VNT = C::VNT, VNCOL = C::VNCOL;
  constexpr int NW = C::NW, NT = C::NT, GW = C::GW, PPW = C::PPW;
  constexpr int VWP = Walsh<VB>::P;
  constexpr int NKIND = VQ ? 2 : 1;
  // weight tasks: (head, TPT consecutive tokens), both kinds; spread over all threads
  constexpr int TPT = (G * kCtaTok) / NT > 0 ? (G * kCtaTok) / NT : 1;
  constexpr int TASKS_PER_HEAD = kCtaTok / TPT;
  constexpr int NTASK = G * TASKS_PER_HEAD;
  static_assert(NTASK <= NT && (TPT == 1 || TPT == 2), "one weight task per thread");
  constexpr int PDB = NKIND * VNCOL * kPdStride;  // one digit buffer (two: current and next)
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ __align__(8) uint64_t mbar[kStagesM + 1];  // per stage (+ one nothing completes: test entry)
  __shared__ int s_fail;                             // a wait of this CTA gave up
  using KL = TileLayout<KB, KQ>;
  using VL = std::conditional_t<KV, KiviVTile, TileLayout<VB, VQ>>;
  constexpr int ktb = KL::BYTES, vtb = VL::BYTES;
  // K stage: the key tile pair, the value norms of its tokens (KIVI: scales), and for KIVI the
  // statistics of the key group the pair starts (when it starts one)
  constexpr int kstage = 2 * ktb + kNormBlock + (KV ? kKiviStats : 0);
  constexpr int stage_bytes = (kstage > 2 * vtb) ? kstage : 2 * vtb;
  // logits row stride (floats): chunk + 8 with the chunk a multiple of 64, so rows start on distinct banks
  const int lgst = p.chunk + 8;
  unsigned char* stages = smem;                                            // [kStagesM][2 tiles (+ norms)]
  float* lgs = reinterpret_cast<float*>(stages + kStagesM * stage_bytes);  // [G][lgst] logits
  unsigned char* pdig = reinterpret_cast<unsigned char*>(lgs + G * lgst);  // [2][NKIND][VNCOL][kPdStride]
  float* red = reinterpret_cast<float*>(pdig + 2 * PDB);                      // reductions
  // KIVI: the query in log2 logit units [G][d]; the current key group's query digits [KP][G][2][d]
  // (bytes; words permuted for load_qb), per head (scale, offset) [G][2]
  float* kq = red + (NW * G + 2 * NW);
  unsigned char* ktab = reinterpret_cast<unsigned char*>(kq + G * kHeadDim);
  float* kcon = reinterpret_cast<float*>(ktab + KP * G * 2 * kHeadDim);

  // One-dimensional grid: the split CTAs (split fastest, then row y, then sequence), then the
  // window parts' CTAs in the same order (mixed-precision caches), which the block scheduler
  // places last: they fill the slots the split CTAs leave free.
  // Row y: piece `half` of kv-head hk's query group (p.hsplit pieces of G heads); a CTA of 8 heads
  // takes the whole group (both prep pieces, one per warp half).
  const int npc = G > 4 ? 1 : p.hsplit;
  const int n_rows = p.Hkv * npc;
  const int n_split_ctas = p.splits * n_rows * p.B;
  const bool win_cta = (int)blockIdx.x >= n_split_ctas;
  const int bx = win_cta ? (int)blockIdx.x - n_split_ctas : (int)blockIdx.x;
  const int nx = win_cta ? p.win_parts : p.splits;
  const int split = bx % nx, row = (bx / nx) % n_rows, b = bx / (nx * n_rows);
  const int hk = row / npc, half = row % npc;
  const int h_first = hk * p.group + half * G;
  if (win_cta) {  // a window part: no staging, no barrier below
    grid_dep_wait();
    window_part<NW, G>(p, b, hk, half * G, split, reinterpret_cast<float*>(smem));
    return;
  }
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hb = G > 4 ? 4 * (warp >> 2) : 0;  // first head of this warp's logits
  const int g = lane >> 2, t = lane & 3;
  // In a fused append + decode step the cache (and len) are written by the append kernel that
  // runs before the prep: everything that reads them waits for the prep (which waits for it).
  const int t_begin = split * p.chunk;
  const size_t pair = (size_t)b * p.Hkv + hk;
  const unsigned char* kreg = reinterpret_cast<const unsigned char*>(p.kreg);
  const unsigned char* vreg = reinterpret_cast<const unsigned char*>(p.vreg);
  // index of a tile pair's first tile (contiguous, or the block table's page)
  // paged caches: the block-table entries of this CTA's chunk, read once into shared memory (the
  // fill issue path then does no global load); chunks are at most kChunkMax tokens
  __shared__ int s_pages[kChunkMax / kCtaTok + 1];
  if (p.table)
    for (int i = threadIdx.x; i <= p.chunk / kCtaTok && (t_begin / kCtaTok + i) < p.pages_per_seq; i += blockDim.x)
      s_pages[i] = __ldcg(p.table + (size_t)b * p.pages_per_seq + t_begin / kCtaTok + i);
  auto pair_index = [&](int tile0) -> long {
    if (!p.table) return ((long)b * p.Hkv + hk) * p.tiles_per_seq + tile0;
    const int page = s_pages[tile0 / 2 - t_begin / kCtaTok];
    if (page < 0 || page >= p.n_pages) {
      atomicOr(p.err, kStatusBadPage);
      return (long)hk * 2;
    }
    return ((long)page * p.Hkv + hk) * 2;
  };
  // In a fused append + decode step the predecessor appends the token at the old length and sets
  // the new one, so a length read before waiting for it is either value. When the first
  // kStagesM - 1 fills end below the old length under both readings, they hold no token the
  // predecessor writes: they are issued before the wait (`early`), the rest after it.
  int len = __ldcg(p.lens + b);  // through L2: a predecessor may write it
  const bool early = p.cache_after_wait && t_begin + kCtaTok * (kStagesM - 1) < len;
  if (p.cache_after_wait && !early) {
    grid_dep_wait();
    len = __ldcg(p.lens + b);
  }
  int t_end = min(len, t_begin + p.chunk);
  int n_iter = t_end > t_begin ? (t_end - t_begin + kCtaTok - 1) / kCtaTok : 0;

  // Staging: fill f < n_iter brings the K tile pair of pass-1 iteration f (and the value norms
  // and sketch norms of the same tokens, for the weight scale); fill n_iter + i brings the V tile
  // pair of pass-2 iteration i. Fill f goes to stage f % kStagesM and completes phase f / kStagesM
  // of that stage's barrier. Thread 0 issues the fills as bulk copies; every tile pair is whole
  // (capacity is a whole number of pairs), so a fill never reads outside its pair's region.
  int n_fill = 2 * n_iter;
  if (tid == 0) {
#pragma unroll
    for (int s = 0; s <= kStagesM; ++s) mbar_init(smem_addr(&mbar[s]), 1);
    mbar_init_fence();
    s_fail = 0;
  }
  __syncthreads();
  auto issue = [&](int f) {  // thread 0 only
    if (f >= n_fill) return;
    const int slot = (unsigned)f % kStagesM;
    const uint32_t bar = smem_addr(&mbar[slot]);
    unsigned char* dst = stages + slot * stage_bytes;
    fence_proxy_async();  // the stage's previous contents were read by the generic proxy
    if (f < n_iter) {
      const long ti = pair_index((unsigned)(t_begin + f * kCtaTok) / kTile);
      constexpr uint32_t nb = VQ ? 128u : 64u;  // value norms (+ gammas, contiguous) per tile
      const int t0 = t_begin + f * kCtaTok;
      const bool stats = KV && t0 % kKiviGroup == 0;  // KIVI: the pair starts a key group
      mbar_arrive_expect_tx(bar, 2u * ktb + 2u * nb + (stats ? (uint32_t)kKiviStats : 0u));
      bulk_g2s(smem_addr(dst), kreg + (size_t)ti * ktb, 2u * ktb, bar);
#pragma unroll
      for (int tile = 0; tile < 2; ++tile)
        bulk_g2s(smem_addr(dst + 2 * ktb + tile * 128), vreg + (size_t)(ti + tile) * vtb + VL::NORM, nb, bar);
      if (stats)
        bulk_g2s(smem_addr(dst + 2 * ktb + kNormBlock),
                 p.kstats + (pair * p.groups_per_seq + t0 / kKiviGroup) * (size_t)kKiviStats, kKiviStats, bar);
    } else {
      const long ti = pair_index((unsigned)(t_begin + (f - n_iter) * kCtaTok) / kTile);
      mbar_arrive_expect_tx(bar, 2u * vtb);
      bulk_g2s(smem_addr(dst), vreg + (size_t)ti * vtb, 2u * vtb, bar);
    }
  };
  auto wait_fill = [&](int f) {  // every thread
    const uint32_t bar = smem_addr(&mbar[(unsigned)f % kStagesM]), par = ((unsigned)f / kStagesM) & 1u;
    if (!mbar_try(bar, par) && !mbar_wait(bar, par, p.wait_limit)) {
      s_fail = 1;
      atomicOr(p.err, 1);
    }
  };
  if (tid == 0)
#pragma unroll
    for (int f = 0; f < kStagesM - 1; ++f) issue(f);  // early: key fills whatever the final length
  if (early) {  // the final length, now that the predecessor has finished
    grid_dep_wait();
    len = __ldcg(p.lens + b);
    t_end = min(len, t_begin + p.chunk);
    n_iter = t_end > t_begin ? (t_end - t_begin + kCtaTok - 1) / kCtaTok : 0;
    n_fill = 2 * n_iter;
  }
  if (p.debug_unset_wait && !mbar_wait(smem_addr(&mbar[kStagesM]), 0u, p.wait_limit)) {
    s_fail = 1;
    atomicOr(p.err, 1);
  }

  // logit-phase B fragments (query digits) and head constants from the prep area (written by the
  // predecessor kernel while this one may already run: loaded through L2, not the read-only path)
  // Launched as a programmatic dependent of the prep kernel: the cache tiles staged above were
  // complete before prep started (unless cache_after_wait, handled above); the prep output is read
  // only after this wait.
  if (!p.cache_after_wait) grid_dep_wait();
  // Query digit table rows: [KP][heads th][2 digits][128 coordinates] bytes from head h_off on (the
  // prep area in global memory, or the KIVI group's table in shared memory)
  uint32_t qb[KP][4][KNT][2];
  auto load_qb = [&](const unsigned char* tab, int th, int h_off) {
#pragma unroll
    for (int P = 0; P < KP; ++P)
#pragma unroll
      for (int nt = 0; nt < KNT; ++nt) {
        const int n = nt * 8 + g, h = n / 2, d = n % 2;  // column = (head of this warp, digit)
        const uint32_t* row = reinterpret_cast<const uint32_t*>(tab + ((P * th + h_off + min(h, GW - 1)) * 2 + d) * 128);
        if constexpr (KV) {  // KIVI's table keeps word x at (x % 4) * 8 + x / 4: two 16-byte loads
          const uint4 w0 = *reinterpret_cast<const uint4*>(row + t * 8);
          const uint4 w1 = *reinterpret_cast<const uint4*>(row + t * 8 + 4);
          const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            qb[P][m][nt][0] = h < GW ? w[2 * m] : 0u;
            qb[P][m][nt][1] = h < GW ? w[2 * m + 1] : 0u;
          }
        } else {
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            qb[P][m][nt][0] = h < GW ? __ldcg(row + (2 * m) * 4 + t) : 0u;
            qb[P][m][nt][1] = h < GW ? __ldcg(row + (2 * m + 1) * 4 + t) : 0u;
          }
        }
      }
  };
  // Rows g, g + 8 of the key contraction carry operand bytes 2^g (g < 7) or -128 (g = 7); the
  // head scales are in units of the -128 byte, so this thread's rows rescale them by rowf.
  const float rowf = g == 7 ? 1.f : -128.f / (float)(1 << g);
  // this thread's logit columns (2t, 2t+1) of N-tile nt: digits (hi, lo) of head 4 nt + t
  float hs[KNT], hc[KNT], hsz[KNT], hcz[KNT];
  if (!KV) {
    const unsigned char* prep = p.qprep + (pair * p.hsplit + (G > 4 ? (warp >> 2) : half)) * p.qprep_stride;
    load_qb(prep, GW, 0);
    const float* hconst = reinterpret_cast<const float*>(prep + KP * GW * 2 * 128);
#pragma unroll
    for (int nt = 0; nt < KNT; ++nt) {
      const int h = min(4 * nt + t, GW - 1);
      hs[nt] = __ldcg(hconst + h * 4 + 0) * rowf;
      hc[nt] = __ldcg(hconst + h * 4 + 1);
      hsz[nt] = __ldcg(hconst + h * 4 + 2) * rowf;
      hcz[nt] = __ldcg(hconst + h * 4 + 3);
    }
  } else {  // KIVI: the query itself; the digits follow per key group
    for (int i = tid; i < G * kHeadDim; i += NT)
      kq[i] = load_q(p.q, ((size_t)b * p.Hq + h_first + i / kHeadDim) * kHeadDim + i % kHeadDim, p.bf16) * p.logit_scale;
    __syncthreads();  // the group builds read other threads' coordinates
  }
  const float vkappa = VQ ? kSqrtHalfPi / (float)p.v.m : 0.f;

  // ================= pass 1: logits of the whole chunk into lgs, running maxima
  float mrow[KNT];  // max over this thread's logits of head 4 nt + t
#pragma unroll
  for (int nt = 0; nt < KNT; ++nt) mrow[nt] = -INFINITY;
  float wmax = 0.f, wmaxz = 0.f;  // largest value weight of each kind seen by this thread
  const int tl = (warp & 3) * 16;
  // chunk maxima per (warp, head): warps write the heads they own, -inf elsewhere
  float* hmax = red;                 // [NW][G]
  float* wred = red + NW * G;        // [2][NW]: both kinds' weight maxima
  for (int i = tid; i < NW * G; i += NT) hmax[i] = -INFINITY;
  for (int it = 0; it < n_iter; ++it) {
    if (tid == 0) issue(it + kStagesM - 1);
    wait_fill(it);
    const unsigned char* kt = stages + ((unsigned)it % kStagesM) * stage_bytes;
    const int tok0 = it * kCtaTok;  // chunk-relative first token of this iteration
    const int count = min(kCtaTok, t_end - (t_begin + tok0));
    if (KV && (t_begin + tok0) % kKiviGroup == 0) {
      // KIVI key group: logit = sum_j q_j (s_j code_j + z_j) with code = b0 + 2 b1, so plane P's
      // query term is 2^P q_j s_j (a 16-bit integer relative to the head's largest |2 q_j s_j|,
      // as two digits) and the head's offset is sum_j q_j z_j. Warp h builds head h: lane l takes
      // coordinates 4l .. 4l + 3, i.e. word x = l of each digit row, stored where load_qb reads it
      // with two 16-byte loads (word x at (x % 4) * 8 + x / 4).
      const __half* st = reinterpret_cast<const __half*>(kt + 2 * ktb + kNormBlock);
      const uint2 s4 = *reinterpret_cast<const uint2*>(st + 4 * lane);
      const uint2 z4 = *reinterpret_cast<const uint2*>(st + kHeadDim + 4 * lane);
      const float2 s01 = __half22float2(*reinterpret_cast<const __half2*>(&s4.x));
      const float2 s23 = __half22float2(*reinterpret_cast<const __half2*>(&s4.y));
      const float2 z01 = __half22float2(*reinterpret_cast<const __half2*>(&z4.x));
      const float2 z23 = __half22float2(*reinterpret_cast<const __half2*>(&z4.y));
      const float sv[4] = {s01.x, s01.y, s23.x, s23.y}, zv[4] = {z01.x, z01.y, z23.x, z23.y};
      const int wpos = (lane & 3) * 8 + (lane >> 2);
      for (int h = warp; h < G; h += NW) {
        const float4 q4 = *reinterpret_cast<const float4*>(kq + h * kHeadDim + 4 * lane);
        const float qv[4] = {q4.x, q4.y, q4.z, q4.w};
        float x[4], a = 0.f, c = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[e] = qv[e] * sv[e];
          a = fmaxf(a, fabsf(x[e]));
          c = fmaf(qv[e], zv[e], c);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
          c += __shfl_xor_sync(0xffffffffu, c, o);
        }
        const float vmax = a > 0.f ? 2.f * a : 1.f;
        const float qsc = (float)kQRange / vmax;
#pragma unroll
        for (int P = 0; P < KP; ++P) {
          uint32_t hw = 0u, lw = 0u;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int q = __float2int_rn(((float)(1 << P) * x[e]) * qsc);
            const int hi = (q + 128) >> 8, lo = q - 256 * hi;
            hw |= (uint32_t)(hi & 0xFF) << (8 * e);
            lw |= (uint32_t)(lo & 0xFF) << (8 * e);
          }
          reinterpret_cast<uint32_t*>(ktab + ((P * G + h) * 2 + 0) * kHeadDim)[wpos] = hw;
          reinterpret_cast<uint32_t*>(ktab + ((P * G + h) * 2 + 1) * kHeadDim)[wpos] = lw;
        }
        if (lane == 0) {
          kcon[2 * h] = vmax / ((float)kQRange * -128.f);
          kcon[2 * h + 1] = c;
        }
      }
      __syncthreads();
      load_qb(ktab, G, hb);
#pragma unroll
      for (int nt = 0; nt < KNT; ++nt) {
        const int h = hb + min(4 * nt + t, GW - 1);
        hs[nt] = kcon[2 * h] * rowf;
        hc[nt] = kcon[2 * h + 1];
      }
    }
    {
      // Key bits in octet order: warp w's tokens 16w..16w+15 are octets o0, o0 + 1 of tile w / 2.
      // Row g of the contraction is token 8 o0 + g, row g + 8 token 8 (o0 + 1) + g: both keep bit g
      // of every byte, so one mask makes an operand register and every value of the row is 2^g
      // (-128 for g = 7), a per-row scale folded into the head constants below.
      const unsigned char* ktile = kt + (tl / kTile) * ktb;
      const int s0 = (tl % kTile) + g, s1 = s0 + 8;
      const int o0 = (tl % kTile) / 8;
      const uint32_t mg = 0x01010101u << g;
      int acc[kKeyChains][KNT][4], accz[kKeyChains][KNT][4];  // independent chains: m % kKeyChains
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int nt = 0; nt < KNT; ++nt)
#pragma unroll
          for (int c = 0; c < 4; ++c) { if (m < kKeyChains) { acc[m][nt][c] = 0; accz[m][nt][c] = 0; } }
      // this thread's words of octet o: 8t + 2m + h, m = 0..3, h = 0..1 (32 contiguous bytes)
      const unsigned char* kp = ktile + KL::PLANES + o0 * 128 + t * 32;
#pragma unroll
      for (int mp = 0; mp < 2; ++mp) {  // coordinate blocks 2 mp, 2 mp + 1: one 16-byte load per octet
        uint4 wa[KB + (KQ ? 1 : 0)], wb[KB + (KQ ? 1 : 0)];  // octets o0, o0 + 1
#pragma unroll
        for (int pp = 0; pp < KB + (KQ ? 1 : 0); ++pp) {
          const int off = (pp < KB ? pp * (kTile * 16) : KL::SKETCH - KL::PLANES) + mp * 16;
          wa[pp] = *reinterpret_cast<const uint4*>(kp + off);
          wb[pp] = *reinterpret_cast<const uint4*>(kp + off + 128);
        }
#pragma unroll
        for (int mm = 0; mm < 2; ++mm) {
          const int m = 2 * mp + mm;
#pragma unroll
          for (int P = 0; P < KP; ++P) {
            const bool sk = KQ && P == KP - 1;
            uint32_t xa0, xa1, xb0, xb1;  // (octet a / b, h = 0 / 1) words of coordinate block m
            auto pick = [&](int pp, uint32_t& a0w, uint32_t& a1w, uint32_t& b0w, uint32_t& b1w) {
              a0w = mm ? wa[pp].z : wa[pp].x; a1w = mm ? wa[pp].w : wa[pp].y;
              b0w = mm ? wb[pp].z : wb[pp].x; b1w = mm ? wb[pp].w : wb[pp].y;
            };
            if (sk) {
              pick(KB, xa0, xa1, xb0, xb1);
            } else if (KB == 3 && P == 3) {  // parity plane
              uint32_t c0, c1, c2, c3;
              pick(0, xa0, xa1, xb0, xb1);
              pick(1, c0, c1, c2, c3);
              xa0 ^= c0; xa1 ^= c1; xb0 ^= c2; xb1 ^= c3;
              pick(KB - 1, c0, c1, c2, c3);
              xa0 ^= c0; xa1 ^= c1; xb0 ^= c2; xb1 ^= c3;
            } else {
              pick(P < KB ? P : 0, xa0, xa1, xb0, xb1);
            }
            const uint32_t a0 = xa0 & mg, a1 = xb0 & mg, a2 = xa1 & mg, a3 = xb1 & mg;
#pragma unroll
            for (int nt = 0; nt < KNT; ++nt) {
              if (sk) mma_s8(accz[m % kKeyChains][nt], a0, a1, a2, a3, qb[P][m][nt][0], qb[P][m][nt][1]);
              else mma_s8(acc[m % kKeyChains][nt], a0, a1, a2, a3, qb[P][m][nt][0], qb[P][m][nt][1]);
            }
          }
        }
      }
      const float nk0 = __half2float(*reinterpret_cast<const __half*>(ktile + KL::NORM + s0 * 2));
      const float nk1 = __half2float(*reinterpret_cast<const __half*>(ktile + KL::NORM + s1 * 2));
      float gk0 = 0.f, gk1 = 0.f;
      if (KQ) {
        gk0 = __half2float(*reinterpret_cast<const __half*>(ktile + KL::GAMMA + s0 * 2));
        gk1 = __half2float(*reinterpret_cast<const __half*>(ktile + KL::GAMMA + s1 * 2));
      }
      const bool v0 = tl + g < count, v1 = tl + g + 8 < count;
#pragma unroll
      for (int nt = 0; nt < KNT; ++nt) {
        const int h = 4 * nt + t;
        int c[4], cz[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          c[e] = acc[0][nt][e];
          cz[e] = accz[0][nt][e];
#pragma unroll
          for (int ch = 1; ch < kKeyChains; ++ch) {
            c[e] += acc[ch][nt][e];
            cz[e] += accz[ch][nt][e];
          }
        }
        // hi * 256 + lo: exact in int32 up to 2 Walsh planes (|hi| < 2^22), else in fp32
        const float c01 = KB <= 2 ? (float)(c[0] * 256 + c[1]) : fmaf((float)c[0], 256.f, (float)c[1]);
        const float c23 = KB <= 2 ? (float)(c[2] * 256 + c[3]) : fmaf((float)c[2], 256.f, (float)c[3]);
        float l0 = fmaf(hs[nt], c01, hc[nt]);
        float l1 = fmaf(hs[nt], c23, hc[nt]);
        if (KQ) {  // one sketch plane: |hi| < 2^21
          l0 = fmaf(gk0, fmaf(hsz[nt], (float)(cz[0] * 256 + cz[1]), hcz[nt]), l0);
          l1 = fmaf(gk1, fmaf(hsz[nt], (float)(cz[2] * 256 + cz[3]), hcz[nt]), l1);
        }
        // (KIVI keys have no per-token norm)
        const float lg0 = v0 ? (KV ? l0 : nk0 * l0) : -INFINITY, lg1 = v1 ? (KV ? l1 : nk1 * l1) : -INFINITY;
        if (h < GW) {
          lgs[(hb + h) * lgst + tok0 + tl + g] = lg0;
          lgs[(hb + h) * lgst + tok0 + tl + g + 8] = lg1;
        }
        mrow[nt] = fmaxf(mrow[nt], fmaxf(lg0, lg1));
      }
    }
    // largest value weight: tokens of this iteration, one per thread of warps 0 and 1
    if (tid < count) {  // staged value norms: [tile][64 B norms | 64 B gammas]
      const unsigned char* nb = kt + 2 * ktb + (tid / kTile) * 128 + (tid % kTile) * 2;
      const float w = __half2float(*reinterpret_cast<const __half*>(nb)) * (KV ? 1.f : kInvSqrtD);
      wmax = fmaxf(wmax, w);
      if (VQ) wmaxz = fmaxf(wmaxz, w * (__half2float(*reinterpret_cast<const __half*>(nb + 64)) * vkappa));
    }
    __syncthreads();  // the next iteration refills a stage buffer
  }
  // chunk maxima per head, and the weight scale
#pragma unroll
  for (int nt = 0; nt < KNT; ++nt) {
    float mx = mrow[nt];
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
    if (g == 0 && 4 * nt + t < GW) hmax[warp * G + hb + 4 * nt + t] = mx;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
    wmaxz = fmaxf(wmaxz, __shfl_xor_sync(0xffffffffu, wmaxz, o));
  }
  if (lane == 0) { wred[warp] = wmax; wred[NW + warp] = wmaxz; }
  for (int idx = tid; idx < 2 * PDB / 4; idx += NT)
    reinterpret_cast<uint32_t*>(pdig)[idx] = 0u;  // the pad digit and absent heads stay zero
  __syncthreads();
  float wm = 0.f, wmz = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) { wm = fmaxf(wm, wred[w]); wmz = fmaxf(wmz, wred[NW + w]); }
  // integer weights below 2^23 (3 byte digits), each kind scaled to its own range by a power
  // of two (exact digits; the sketch weights are ~sqrt(pi/2) gamma / m of the centroid ones)
  const float wsc = wm > 0.f ? exp2f(floorf(log2f(kWRange / wm)) - 1.f) : 1.f;
  const float wscz = wmz > 0.f ? exp2f(floorf(log2f(kWRange / wmz)) - 1.f) : 1.f;

  // ================= pass 2: weights -> digits, value contractions
  const bool has_task = tid < NTASK;
  const int task_h = min(tid / TASKS_PER_HEAD, G - 1), task_T = TPT * (tid % TASKS_PER_HEAD);
  float task_m = -INFINITY;
#pragma unroll
  for (int w = 0; w < NW; ++w) task_m = fmaxf(task_m, hmax[w * G + task_h]);
  float task_l = 0.f;                 // sum of p over this task's tokens
  uint32_t task_wc = 0, task_wz = 0;  // sums of the quantised weights (exact: <= 64 tokens x 2^23)
  float task_pz = 0.f;                // KIVI: sum of p z over this task's tokens (value zero points)

  // Weight digits of pass-2 iteration `it` into digit buffer it & 1: p = 2^(l - m) for the task's
  // tokens, then both kinds of value weight; w * scale is rounded by adding 2^23, after which the
  // float's low three bytes are the integer, i.e. directly its three byte digits. Tokens past the
  // end have logit -inf (p = 0) and their norms are masked (a tile's tail may hold anything).
  // Reads the logits and the value norms of fill n_iter + it (which must have landed).
  auto tasks = [&](int it) {
    if (!has_task) return;
    const int tok0 = it * kCtaTok, T = task_T;
    const int count = min(kCtaTok, t_end - (t_begin + tok0));
    const unsigned char* vtile = stages + ((unsigned)(n_iter + it) % kStagesM) * stage_bytes + ((unsigned)T / kTile) * vtb;
    float lv[TPT], wc[TPT], wz[TPT];
    if (TPT == 2) {
      const float2 l2 = *reinterpret_cast<const float2*>(lgs + task_h * lgst + tok0 + T);
      const float2 n2 = __half22float2(*reinterpret_cast<const __half2*>(vtile + VL::NORM + ((unsigned)T % kTile) * 2));
      lv[0] = l2.x; lv[TPT - 1] = l2.y; wc[0] = n2.x; wc[TPT - 1] = n2.y;
      if (VQ || KV) {
        const float2 g2 = __half22float2(*reinterpret_cast<const __half2*>(vtile + VL::GAMMA + ((unsigned)T % kTile) * 2));
        wz[0] = g2.x; wz[TPT - 1] = g2.y;
      }
    } else {
      lv[0] = lgs[task_h * lgst + tok0 + T];
      wc[0] = __half2float(*reinterpret_cast<const __half*>(vtile + VL::NORM + ((unsigned)T % kTile) * 2));
      if (VQ || KV) wz[0] = __half2float(*reinterpret_cast<const __half*>(vtile + VL::GAMMA + ((unsigned)T % kTile) * 2));
    }
    uint32_t bc[TPT], bz[TPT];
    float psum = 0.f;
#pragma unroll
    for (int e = 0; e < TPT; ++e) {
      const bool ok = T + e < count;
      const float pe = ex2(lv[e] - task_m);
      psum += pe;
      const float n = ok ? wc[e] * ((KV ? 1.f : kInvSqrtD) * wsc) : 0.f;
      bc[e] = __float_as_uint(fmaf(pe, n, kRoundBias));
      task_wc += bc[e] - 0x4B000000u;
      if (KV && ok) task_pz = fmaf(pe, wz[e], task_pz);
      if (VQ) {
        const float nz = ok ? wc[e] * wz[e] * (kInvSqrtD * wscz * vkappa) : 0.f;
        bz[e] = __float_as_uint(fmaf(pe, nz, kRoundBias));
        task_wz += bz[e] - 0x4B000000u;
      }
    }
    task_l += psum;
    unsigned char* col = pdig + (it & 1) * PDB + (size_t)(3 * task_h) * kPdStride + T;
#pragma unroll
    for (int kind = 0; kind < NKIND; ++kind) {
      const uint32_t* bw = kind ? bz : bc;
      unsigned char* ck = col + (size_t)kind * VNCOL * kPdStride;
      if (TPT == 2) {  // digit rows 0, 1, 2 = bytes 2, 1, 0 of the rounded floats
        *reinterpret_cast<uint16_t*>(ck) = (uint16_t)__byte_perm(bw[0], bw[TPT - 1], 0x62);
        *reinterpret_cast<uint16_t*>(ck + kPdStride) = (uint16_t)__byte_perm(bw[0], bw[TPT - 1], 0x51);
        *reinterpret_cast<uint16_t*>(ck + 2 * kPdStride) = (uint16_t)__byte_perm(bw[0], bw[TPT - 1], 0x40);
      } else {
        ck[0] = (unsigned char)(bw[0] >> 16);
        ck[kPdStride] = (unsigned char)(bw[0] >> 8);
        ck[2 * kPdStride] = (unsigned char)bw[0];
      }
    }
  };

  int vacc[VP][PPW][VNT][4];
#pragma unroll
  for (int P = 0; P < VP; ++P)
#pragma unroll
    for (int pi = 0; pi < PPW; ++pi)
#pragma unroll
      for (int nt = 0; nt < VNT; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) vacc[P][pi][nt][c] = 0;
  const uint32_t vm0 = 0x01010101u << (PPW * warp), vm1 = 0x01010101u << (PPW * warp + PPW - 1);

  // Digits of iteration 0, then per iteration: the digits of the next one (all threads) and the
  // contractions of this one; one barrier per iteration separates the two digit buffers.
  if (n_iter > 0) {
    wait_fill(n_iter);
    tasks(0);
  }
  __syncthreads();
  for (int it = 0; it < n_iter; ++it) {
    if (tid == 0) issue(n_iter + it + kStagesM - 1);
    if (it + 1 < n_iter) {
      wait_fill(n_iter + it + 1);
      tasks(it + 1);
    }
    const unsigned char* vt = stages + ((unsigned)(n_iter + it) % kStagesM) * stage_bytes;
    const unsigned char* pd = pdig + (it & 1) * PDB;

    // value contractions: positions 2w, 2w+1 of every value Walsh plane
#pragma unroll
    for (int s = 0; s < 2; ++s) {  // a step past the end adds nothing: its weights are zero
      const unsigned char* vtile = vt + s * vtb;
      // K order within a 32-token step: K-index 4t + i <-> token 8t + i, 16 + 4t + i <-> 8t + 4 + i,
      // so a thread's two 4-token groups are one 64-bit load (bits and digits alike)
      uint32_t bm[VNT][2], bz[VNT][2];
#pragma unroll
      for (int nt = 0; nt < VNT; ++nt) {
        const unsigned char* col = pd + (size_t)(nt * 8 + g) * kPdStride + s * kTile + 8 * t;
        const uint2 v = *reinterpret_cast<const uint2*>(col);
        bm[nt][0] = v.x;
        bm[nt][1] = v.y;
        if (VQ) {
          const uint2 vz = *reinterpret_cast<const uint2*>(col + (size_t)VNCOL * kPdStride);
          bz[nt][0] = vz.x;
          bz[nt][1] = vz.y;
        }
      }
      uint32_t xv[4][4];  // code planes, then the sketch plane (same byte-lane-major layout)
#pragma unroll
      for (int pp = 0; pp < VB + (VQ ? 1 : 0); ++pp) {
        const unsigned char* pl =
            vtile + (pp < VB ? VL::PLANES + pp * (kTile * 16) : VL::SKETCH) + 8 * t;
        const uint2 r0 = *reinterpret_cast<const uint2*>(pl + g * kTile);
        const uint2 r1 = *reinterpret_cast<const uint2*>(pl + (g + 8) * kTile);
        xv[pp][0] = r0.x; xv[pp][2] = r0.y;
        xv[pp][1] = r1.x; xv[pp][3] = r1.y;
      }
#pragma unroll
      for (int P = 0; P < VP; ++P) {
        const bool sk = VQ && P == VP - 1;
        uint32_t x[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          if (sk) {
            x[r] = xv[VB][r];
          } else if (VB == 3 && P == 3) {
            x[r] = xv[0][r] ^ xv[1][r] ^ xv[2][r];
          } else {
            x[r] = xv[P][r];
          }
        }
        const uint32_t a00 = x[0] & vm0, a01 = x[1] & vm0, a02 = x[2] & vm0, a03 = x[3] & vm0;
        const uint32_t a10 = x[0] & vm1, a11 = x[1] & vm1, a12 = x[2] & vm1, a13 = x[3] & vm1;
#pragma unroll
        for (int nt = 0; nt < VNT; ++nt) {
          const uint32_t b0 = sk ? bz[nt][0] : bm[nt][0], b1 = sk ? bz[nt][1] : bm[nt][1];
          mma_s8u8(vacc[P][0][nt], a00, a01, a02, a03, b0, b1);
          if (PPW > 1) mma_s8u8(vacc[P][PPW - 1][nt], a10, a11, a12, a13, b0, b1);
        }
      }
    }
    __syncthreads();  // the next iteration refills a stage buffer and the digits
  }

  grid_dep_launch();  // let the split reduce be scheduled; it waits for this grid to finish
  // ================= finish: per-head sums of p and of the weights, then this warp's rows
  // Every fill was waited for above; after a wait that gave up, thread 0 waits once more (bounded)
  // for the last fill of each stage, so no copy is still landing when the stages are reused.
  if (tid == 0 && s_fail)
    for (int f = max(0, n_fill - kStagesM); f < n_fill; ++f)
      mbar_wait(smem_addr(&mbar[(unsigned)f % kStagesM]), ((unsigned)f / kStagesM) & 1u, p.wait_limit);
  __syncthreads();
  float* tsum = reinterpret_cast<float*>(stages);  // [NT][3] (staging reused)
  float* hsum = tsum + 3 * NT;                      // [3][G]: sum p, sum weights, sum sketch weights
  tsum[3 * tid] = task_l;
  tsum[3 * tid + 1] = (float)task_wc;
  tsum[3 * tid + 2] = KV ? task_pz : (float)task_wz;
  __syncthreads();
  if (tid < 3 * G) {
    const int what = tid / G, h = tid % G;  // what: 0 sum p, 1 sum weights, 2 sum sketch weights (KIVI: p z)
    float s2 = 0.f;
    for (int q = 0; q < TASKS_PER_HEAD; ++q) s2 += tsum[3 * (h * TASKS_PER_HEAD + q) + what];
    hsum[tid] = s2;
  }
  __syncthreads();
  float va[4];
  walsh_coeffs(VB, p.v.cent, va);
  float vasum = 0.f;
#pragma unroll
  for (int P = 0; P < VWP; ++P) vasum += va[P];
  if (KV) {  // KIVI codes b0 + 2 b1 on 0/1 planes: 2 va_P = 2^P, no Walsh offset
    va[0] = 0.5f;
    va[1] = 1.f;
    vasum = 0.f;
  }
  const float inv_w = 1.f / wsc, inv_wz = 1.f / wscz;
  // Column c = 3h + d of the value contraction holds byte digit d (weight 2^16, 2^8, 1) of head h,
  // on lane 4g + (c % 8) / 2 (register pair c / 8, element c % 2): the quad of lanes 4g .. 4g + 3
  // holds every column of rows g and g + 8, so each head's three digits are gathered by shuffles
  // (a fixed summation order) and lane 4g + h % 4 writes the head's coordinates.
  float offs[G], offz[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    offs[h] = KV ? hsum[2 * G + h] : -vasum * hsum[G + h] * inv_w;  // KIVI: sum_t p_t z_t
    offz[h] = VQ ? -hsum[2 * G + h] * inv_wz : 0.f;
  }
#pragma unroll
  for (int pi = 0; pi < PPW; ++pi) {
    const int pos = PPW * warp + pi;
    const float rowpos = pos == 7 ? -1.f / 128.f : 1.f / (float)(1 << pos);  // row value 2^p or -128
    const float rowinv = rowpos * inv_w, rowinvz = rowpos * inv_wz;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int j = 8 * (g + 8 * rr) + pos;  // coordinate of row g (rr = 0) or g + 8
      float vo[VNT][2], vz[VNT][2];  // this lane's columns, planes folded
#pragma unroll
      for (int nt = 0; nt < VNT; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float o = 0.f, z = 0.f;
#pragma unroll
          for (int P = 0; P < VP; ++P) {
            const float r = (float)vacc[P][pi][nt][2 * rr + e];
            if (VQ && P == VP - 1) z = 2.f * r;
            else o = fmaf(2.f * va[min(P, 3)], r, o);
          }
          vo[nt][e] = o;
          vz[nt][e] = z;
        }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float dg[3], dz[3];
#pragma unroll
        for (int d = 0; d < 3; ++d) {
          const int c = 3 * h + d, src = (lane & ~3) | ((c & 7) >> 1);
          dg[d] = __shfl_sync(0xffffffffu, vo[c >> 3][c & 1], src);
          if (VQ) dz[d] = __shfl_sync(0xffffffffu, vz[c >> 3][c & 1], src);
        }
        if ((lane & 3) == (h & 3)) {
          float* dst = p.part + (((size_t)b * p.Hq + h_first + h) * p.splits + split) * p.part_stride;
          dst[2 + j] = fmaf(fmaf(dg[0], 65536.f, dg[1] * 256.f) + dg[2], rowinv, offs[h]);
          if (VQ) dst[2 + kHeadDim + j] = fmaf(fmaf(dz[0], 65536.f, dz[1] * 256.f) + dz[2], rowinvz, offz[h]);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (tid == h) {
      float* dst = p.part + (((size_t)b * p.Hq + h_first + h) * p.splits + split) * p.part_stride;
      float mx = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) mx = fmaxf(mx, hmax[w * G + h]);
      dst[0] = mx;
      dst[1] = hsum[h];
    }
  }

}

// Query prep of a decode call, or the fused step's front kernel (append + query prep) when qp is given.
template <int G, int KB, bool KQ>
cudaError_t launch_prep(const DecodeParams& p, cudaStream_t s, const QuantizeParams* qp) {
  const size_t prep_smem = KQ ? sizeof(float) * kHeadDim * kHeadDim : 0;
  cudaError_t e = cudaFuncSetAttribute(decode_lm_prep<G, KB, KQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)prep_smem);
  if (e != cudaSuccess) return e;
  if (qp) {  // fused step: append + prep in one launch
    const int nq = qlm::blocks_per_side(*qp);
    const size_t fsmem = std::max(prep_smem, (size_t)sizeof(float) * kHeadDim * kHeadDim);
    e = cudaFuncSetAttribute(decode_front<G, KB, KQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)fsmem);
    if (e != cudaSuccess) return e;
    // a programmatic dependent of whatever precedes it: its launch and setup overlap that
    // kernel's tail, and it waits for it before reading inputs
    cudaLaunchConfig_t fc = {};
    fc.gridDim = dim3(2 * nq + p.B * p.Hkv * p.hsplit);
    fc.blockDim = dim3(kThreadsM);
    fc.dynamicSmemBytes = fsmem;
    fc.stream = s;
    cudaLaunchAttribute fa[1];
    fa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    fa[0].val.programmaticStreamSerializationAllowed = 1;
    fc.attrs = fa;
    fc.numAttrs = 1;
    e = cudaLaunchKernelEx(&fc, decode_front<G, KB, KQ>, *qp, p, nq);
    if (e != cudaSuccess) return e;
  } else {
    decode_lm_prep<G, KB, KQ><<<dim3(p.Hkv * p.hsplit, p.B), kThreadsM, prep_smem, s>>>(p);
  }
  return launched();
}

template <int G, int KB, bool KQ, int VB, bool VQ, bool KV = false>
cudaError_t launch_mma(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  using VL = std::conditional_t<KV, KiviVTile, TileLayout<VB, VQ>>;
  if (!TileLayout<KB, KQ>::matches(p.k) || !VL::matches(p.v)) return cudaErrorNotSupported;
  if (p.k.order != kOrderOctet || p.v.order != kOrderByteLane) return cudaErrorNotSupported;
  if (KV && (p.chunk % kKiviGroup || qp)) return cudaErrorNotSupported;  // whole key groups per CTA
  cudaError_t e = cudaSuccess;
  // query prep in pieces of <= 4 heads (KIVI: none; the CTAs build each key group's digits)
  if (!KV && (e = launch_prep<(G > 4 ? 4 : G), KB, KQ>(p, s, qp)) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  size_t smem = mma_smem_bytes(G, p.k, p.v, p.chunk, KV);
  if (p.win_fused) smem = std::max(smem, sizeof(float) * window_smem_floats<MmaCfg<G, KB, KQ, VB, VQ>::NW, G>());
  auto kern = decode_lm_mma<G, KB, KQ, VB, VQ, KV>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  // split CTAs, then the window parts' CTAs (mixed-precision caches), in one dimension
  const long rows = (long)p.Hkv * (G > 4 ? 1 : p.hsplit) * p.B;
  const long ctas = rows * (p.splits + (p.win_fused ? p.win_parts : 0));
  if (ctas > 0x7fffffffL) return cudaErrorInvalidValue;
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(MmaCfg<G, KB, KQ, VB, VQ>::NT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return e;
  return launched();
}

template <int G>
cudaError_t dispatch_mma_modes(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  const int kb = p.k.bits, vb = p.v.bits;
  const bool kq = p.k.qjl, vq = p.v.qjl;
#define KVQ_MMA_CASE(KB, KQ, VB, VQ) \
  if (kb == KB && kq == KQ && vb == VB && vq == VQ) return launch_mma<G, KB, KQ, VB, VQ>(p, s, ev_mid, qp);
  KVQ_MMA_CASE(2, true, 2, true)
  KVQ_MMA_CASE(3, true, 3, false)
  KVQ_MMA_CASE(1, false, 1, false)
  KVQ_MMA_CASE(2, true, 2, false)
  KVQ_MMA_CASE(3, true, 3, true)
  KVQ_MMA_CASE(2, false, 2, false)
  KVQ_MMA_CASE(3, false, 3, false)
#undef KVQ_MMA_CASE
  return cudaErrorNotSupported;
}

template <int G>
cudaError_t dispatch_prep(const DecodeParams& p, cudaStream_t s, const QuantizeParams* qp) {
  const int kb = p.k.bits;
  const bool kq = p.k.qjl;
  if (kb == 1 && !kq) return launch_prep<G, 1, false>(p, s, qp);
  if (kb == 2 && kq) return launch_prep<G, 2, true>(p, s, qp);
  if (kb == 2 && !kq) return launch_prep<G, 2, false>(p, s, qp);
  if (kb == 3 && kq) return launch_prep<G, 3, true>(p, s, qp);
  if (kb == 3 && !kq) return launch_prep<G, 3, false>(p, s, qp);
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_lm_query_prep(const DecodeParams& p, cudaStream_t s, const QuantizeParams* qp) {
  switch (p.group / p.hsplit) {  // heads of one prep piece
    case 1: return dispatch_prep<1>(p, s, qp);
    case 2: return dispatch_prep<2>(p, s, qp);
    case 4: return dispatch_prep<4>(p, s, qp);
    default: return cudaErrorNotSupported;
  }
}

int mma_prep_bytes(int k_bits, int k_qjl, int group) {
  const int kp = (k_bits == 3 ? 4 : k_bits) + (k_qjl ? 1 : 0);
  const int bytes = kp * group * 2 * 128 + 16 * group;
  return (bytes + 255) / 256 * 256;
}

bool mma_modes_supported(int group, int k_bits, int k_qjl, int v_bits, int v_qjl) {
  if (group != 1 && group != 2 && group != 4 && group != 8) return false;
  // the (K bits, K sketch, V bits, V sketch) instances of dispatch_mma_modes
  static const int kModes[][4] = {{2, 1, 2, 1}, {3, 1, 3, 0}, {1, 0, 1, 0}, {2, 1, 2, 0},
                                  {3, 1, 3, 1}, {2, 0, 2, 0}, {3, 0, 3, 0}};
  for (const auto& m : kModes)
    if (m[0] == k_bits && m[1] == (k_qjl ? 1 : 0) && m[2] == v_bits && m[3] == (v_qjl ? 1 : 0)) return true;
  return false;
}

// Resident CTAs per SM of one instance as its registers and threads allow (shared memory aside),
// from the runtime's occupancy calculator, once per instance.
template <int G, int KB, bool KQ, int VB, bool VQ, bool KV>
int mma_reg_slots() {
  static int slots = 0;
  if (slots == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_lm_mma<G, KB, KQ, VB, VQ, KV>,
                                                      MmaCfg<G, KB, KQ, VB, VQ>::NT, 0) != cudaSuccess || n < 1)
      n = 16 / MmaCfg<G, KB, KQ, VB, VQ>::NW;  // the launch bounds' guarantee
    slots = n;
  }
  return slots;
}

template <int G>
int mma_reg_slots_modes(const SideLayout& k, const SideLayout& v, bool kivi) {
  if (kivi) return mma_reg_slots<G, 2, false, 2, false, true>();
#define KVQ_SLOTS_CASE(KB, KQ, VB, VQ) \
  if (k.bits == KB && k.qjl == KQ && v.bits == VB && v.qjl == VQ) return mma_reg_slots<G, KB, KQ, VB, VQ, false>();
  KVQ_SLOTS_CASE(2, true, 2, true)
  KVQ_SLOTS_CASE(3, true, 3, false)
  KVQ_SLOTS_CASE(1, false, 1, false)
  KVQ_SLOTS_CASE(2, true, 2, false)
  KVQ_SLOTS_CASE(3, true, 3, true)
  KVQ_SLOTS_CASE(2, false, 2, false)
  KVQ_SLOTS_CASE(3, false, 3, false)
#undef KVQ_SLOTS_CASE
  return 16 / Warps<G>::N;
}

int lm_mma_slots_per_sm(int group, const SideLayout& k, const SideLayout& v, int chunk, bool kivi) {
  const size_t per = mma_smem_bytes(group, k, v, chunk, kivi) + kSmemReserved;
  int by_regs = 16 / Warps<8>::N;
  switch (group) {
    case 1: by_regs = mma_reg_slots_modes<1>(k, v, kivi); break;
    case 2: by_regs = mma_reg_slots_modes<2>(k, v, kivi); break;
    case 4: by_regs = mma_reg_slots_modes<4>(k, v, kivi); break;
    case 8: by_regs = mma_reg_slots_modes<8>(k, v, kivi); break;
    default: break;
  }
  return std::max(1, std::min(by_regs, (int)(kSmemPerSm / per)));
}

bool mma_decode_supported(const DecodeParams& p) {
  if (!mma_modes_supported(p.group, p.k.bits, p.k.qjl, p.v.bits, p.v.qjl) || p.k.order != kOrderOctet) return false;
  return (p.group == 1 || p.group == 2 || p.group == 4 || (p.group == 8 && p.hsplit == 2)) && p.chunk % kCtaTok == 0 &&
         p.chunk <= kChunkMax && p.qprep != nullptr;
}

cudaError_t launch_decode_kivi_mma(const DecodeParams& p, cudaStream_t s) {
  switch (p.group) {
    case 1: return launch_mma<1, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    case 2: return launch_mma<2, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    case 4: return launch_mma<4, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    case 8: return launch_mma<8, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_decode_lm_mma(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  switch (p.group) {
    case 1: return dispatch_mma_modes<1>(p, s, ev_mid, qp);
    case 2: return dispatch_mma_modes<2>(p, s, ev_mid, qp);
    case 4: return dispatch_mma_modes<4>(p, s, ev_mid, qp);
    case 8: return dispatch_mma_modes<8>(p, s, ev_mid, qp);  // one CTA of 8 warps per kv-head
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kvq
