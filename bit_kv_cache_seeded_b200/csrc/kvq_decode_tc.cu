// Split-K decode attention for LM / LM_QJL / SIGN1 caches on the 5th-generation tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory), one CTA per (sequence, kv-head, split)
// with every query head of the group.
//
// Same computation and the same integer formulation as the mma.sync kernel (kvq_decode_mma.cu;
// "TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and OSCAR": logits
// from the Lloyd-Max centroids plus the unbiased QJL correction, softmax, values dequantised on
// the fly), with the contractions moved to tcgen05:
//   * Logits, per 128-token iteration: D_k [128 tokens x 16] = A [128 tokens x 128 KP] . B_k.
//     A is the key bits expanded to bytes, written by the CTA's threads straight into tensor memory
//     (row = token = lane; a thread masks bit j of every byte of its octet's words, giving the u8
//     value 2^j, a per-row power of two folded into the head scales); its K order is the octet
//     words' byte order, so B_k -- the query digits of every Walsh plane, 16-bit integer terms as two
//     s8 digit columns per head -- is staged once per CTA in shared memory in that order.
//     The sketch plane has its own accumulator (its per-token scale is the residual norm).
//   * Values: D_v[P] [128 coordinates x N] += A [128 coordinates x 128 tokens] . B_v, one accumulator
//     per Walsh plane (and the value sketch plane), kept in tensor memory over the whole chunk. A is
//     the value bits of coordinate row j = 8k + p (byte lane k, bit p: u8 value 2^p) for 128 tokens;
//     B_v is the softmax weights p_t n_t / sqrt(d) (sketch plane: times sqrt(pi/2)/m gamma_t) as
//     23-bit integers in three u8 digit columns per head, built per iteration in shared memory.
//   * Two passes over the chunk, as in the mma.sync kernel: pass 1 writes every logit of the chunk
//     to shared memory and finds the maxima; pass 2 uses fixed weights 2^(l - M), so the integer
//     accumulators are exact and never rescaled.
// CTA: 8 warps, one CTA per SM (512 tensor-memory columns). Warp w reaches tensor-memory lanes
// 32 (w % 4) .. +31 (its quarter's tokens in pass 1, coordinates in pass 2); warps w and w + 4 split
// the planes of those rows between them. Per iteration: every thread expands its planes into one of
// two A buffers (tcgen05.st), a CTA barrier, thread 0 issues the MMAs and commits them to an
// mbarrier, and while they run the threads finish the previous iteration (pass 1: read its logit
// accumulators). Cache tiles arrive by bulk copies (TMA 1-D) into four shared-memory stages, as in
// the mma.sync kernel. Every wait is bounded; a wait that gives up sets bit 0 of the cache's status
// word, and the kernel still runs to its end after waiting (bounded) for its own MMAs and copies.
// Partials (m, l, o_r, acc_z) are written in the format of the other LM kernels; the same reduce
// kernel finishes.
#include <algorithm>
#include <type_traits>

#include <cuda_fp16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_lm_common.cuh"
#include "kvq_tcgen05.cuh"
#include "kvq_tiles.cuh"

namespace kvq {
namespace {

using namespace lmc;

constexpr int kThreadsT = 256;
constexpr int kTokT = 128;             // tokens per iteration (four cache tiles)
constexpr int kStagesT = 4;            // bulk-copy stages
constexpr uint32_t kTmemColsT = 512;
constexpr int kNormBlockT = 4 * 128;   // staged value norms (+ residual norms) of four tiles
constexpr int kKN = 16;                // key-phase N: (head, digit) columns, padded


// KV: the KIVI instance (2-bit unsigned codes b0 + 2 b1 instead of Walsh planes; per-group query
// digits; per-token value scale and zero; no rotation).
template <int G, int KB, bool KQ, int VB, bool VQ, bool KV = false>
struct TcCfg {
  static constexpr int KWP = Walsh<KB>::P, KP = KWP + (KQ ? 1 : 0);  // key planes (sketch last)
  static constexpr int VWP = Walsh<VB>::P, VP = VWP + (VQ ? 1 : 0);  // value planes (sketch last)
  static constexpr int NKIND = VQ ? 2 : 1;
  static constexpr int NK0 = ((3 * G + 15) / 16) * 16;  // value-phase N per kind: (head, digit)
  static constexpr int VN = NKIND * NK0;                // rows of B_v
  static constexpr int APL = KP > VP ? KP : VP;         // planes of one A buffer (32 columns each)
  static constexpr int NBUF = (2 * APL * 32 + 4 * kKN + VP * NK0 <= (int)kTmemColsT) ? 2 : 1;
  static constexpr uint32_t COL_A = 0;                              // buffer a: COL_A + a * APL * 32
  static constexpr uint32_t COL_DK = NBUF * APL * 32;               // [2][main kKN | sketch kKN]
  static constexpr uint32_t COL_DV = COL_DK + 4 * kKN;              // [VP][NK0]
  static_assert(COL_DV + VP * NK0 <= kTmemColsT, "tensor memory");
  static constexpr int GH = (G + 1) / 2;                // heads per warp half in the epilogues
  static constexpr int TPT = G >= 2 ? G / 2 : 1;        // tokens per weight task
  static constexpr int NTASK = G * kTokT / TPT;         // weight tasks per iteration (<= threads)
  static_assert(NTASK <= kThreadsT && TPT <= 4, "one weight task per thread");
  using KL = TileLayout<KB, KQ>;
  using VL = std::conditional_t<KV, KiviVTile, TileLayout<VB, VQ>>;
  static constexpr int KSTAGE = 4 * KL::BYTES + kNormBlockT + (KV ? kKiviStats : 0);
  static constexpr int STAGE = ((KSTAGE > 4 * VL::BYTES ? KSTAGE : 4 * VL::BYTES) + 127) / 128 * 128;
  // query digits: [KP][16 rows][128 K bytes] core matrices (KIVI: two buffers, rebuilt per group)
  static constexpr int BK = (KV ? 2 : 1) * KP * kKN * 128;
  static constexpr int BV = VN * kTokT;      // one weight-digit buffer: [VN rows][128 tokens]
};

// Row stride (floats) of the logits buffer: the chunk rounded up to whole iterations, plus 8 so
// that rows start on distinct banks.
__host__ __device__ inline int tc_logit_stride(int chunk) { return (chunk + kTokT - 1) / kTokT * kTokT + 8; }

// Dynamic shared memory: stages | B_k | 2 x B_v | logits [G][stride] | reductions.
template <class C>
size_t tc_smem_bytes(int G, int chunk) {
  return (size_t)kStagesT * C::STAGE + C::BK + 2 * C::BV + sizeof(float) * (size_t)G * tc_logit_stride(chunk) +
         sizeof(float) * (size_t)(8 * G + 16 + 4 * kThreadsT) + sizeof(float) * (size_t)G * (kHeadDim + 4 + 24);
}

// Byte offset of (row n, K index k) in a K-major operand of core matrices with `kchunks` 16-byte K
// chunks per 8-row group: core (n / 8, k / 16) at ((n / 8) * kchunks + k / 16) * 128.
__device__ __forceinline__ int core_off(int n, int k, int kchunks) {
  return ((n >> 3) * kchunks + (k >> 4)) * 128 + (n & 7) * 16 + (k & 15);
}

template <int G, int KB, bool KQ, int VB, bool VQ, bool KV>
__global__ void __launch_bounds__(kThreadsT, 1) decode_lm_tc(const __grid_constant__ DecodeParams p) {
  using C = TcCfg<G, KB, KQ, VB, VQ, KV>;
  using KL = typename C::KL;
  using VL = typename C::VL;
  constexpr int KP = C::KP, KWP = C::KWP, VP = C::VP, VWP = C::VWP, NK0 = C::NK0, GH = C::GH, TPT = C::TPT;
  constexpr int ktb = KL::BYTES, vtb = VL::BYTES;
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t fill_bar[kStagesT + 1];  // per stage (+ one nothing completes: test entry)
  __shared__ __align__(8) uint64_t mma_bar[2];              // MMA group g commits to mma_bar[g & 1]
  __shared__ uint32_t s_tmem;
  __shared__ int s_fail;

  const int lgst = tc_logit_stride(p.chunk);
  unsigned char* stages = smem;
  unsigned char* bk = stages + kStagesT * C::STAGE;
  unsigned char* bv = bk + C::BK;
  float* lgs = reinterpret_cast<float*>(bv + 2 * C::BV);
  float* red = lgs + G * lgst;  // [8][G] maxima | [16] weight maxima | [4][threads] task sums
  // KIVI: q * scale * log2(e) [G][d], per-iteration head scales and offsets [2][G] each, reductions [8][G] x 2
  float* qsm = red + 8 * G + 16 + 4 * kThreadsT;
  float* hsk = qsm + G * kHeadDim;
  float* hck = hsk + 2 * G;
  float* kred = hck + 2 * G;

  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int qtr = warp & 3, hf = warp >> 2;
  const int t_begin = split * p.chunk;
  const size_t pair = (size_t)b * p.Hkv + hk;
  const int h_first = hk * p.group;
  const unsigned char* kreg = reinterpret_cast<const unsigned char*>(p.kreg);
  const unsigned char* vreg = reinterpret_cast<const unsigned char*>(p.vreg);
  // index of a tile pair's first tile (contiguous, or the block table's page)
  auto pair_index = [&](int tile0) {
    return tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk, tile0, p.err);
  };
  // fused append + decode step: see decode_lm_mma (a length read before the wait is either value)
  int len = __ldcg(p.lens + b);
  const bool early = p.cache_after_wait && t_begin + kTokT * (kStagesT - 1) < len;
  if (p.cache_after_wait && !early) {
    grid_dep_wait();
    len = __ldcg(p.lens + b);
  }
  int t_end = min(len, t_begin + p.chunk);
  int n_iter = t_end > t_begin ? (t_end - t_begin + kTokT - 1) / kTokT : 0;
  int n_fill = 2 * n_iter;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s <= kStagesT; ++s) mbar_init(smem_addr(&fill_bar[s]), 1);
    mbar_init(smem_addr(&mma_bar[0]), 1);
    mbar_init(smem_addr(&mma_bar[1]), 1);
    mbar_init_fence();
    s_fail = 0;
  }
  if (warp == 0) tc::alloc(smem_addr(&s_tmem), kTmemColsT);
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t trow = tmem + ((uint32_t)(32 * qtr) << 16);  // this warp's lane quarter

  // Fill f < n_iter: the K tiles of pass-1 iteration f (whole tile pairs that hold tokens below
  // t_end) and the value norms of the same tiles; fill n_iter + i: the V tiles of pass-2 iteration
  // i. Fill f goes to stage f % kStagesT, completing phase f / kStagesT of its barrier.
  auto issue = [&](int f) {  // thread 0 only
    if (f >= n_fill) return;
    const int slot = (unsigned)f % kStagesT;
    const uint32_t bar = smem_addr(&fill_bar[slot]);
    unsigned char* dst = stages + slot * C::STAGE;
    const int it = f < n_iter ? f : f - n_iter;
    const int t0 = t_begin + it * kTokT;
    const int tile0 = (unsigned)t0 / kTile;
    const int npairs = min(2, (t_end - t0 + 2 * kTile - 1) / (2 * kTile));  // tile pairs with tokens
    fence_proxy_async();  // the stage's previous contents were read by the generic proxy
    if (f < n_iter) {
      constexpr uint32_t nb = VQ ? 128u : 64u;  // value norms (+ gammas, contiguous) per tile
      mbar_arrive_expect_tx(bar, (uint32_t)npairs * 2u * (ktb + nb) + (KV ? (uint32_t)kKiviStats : 0u));
      if (KV)  // the key group's statistics (iterations are whole 128-token groups)
        bulk_g2s(smem_addr(dst + 4 * ktb + kNormBlockT),
                 p.kstats + (pair * p.groups_per_seq + (unsigned)t0 / kTokT) * (size_t)kKiviStats, kKiviStats, bar);
      for (int j = 0; j < npairs; ++j) {
        const long ti = pair_index(tile0 + 2 * j);
        bulk_g2s(smem_addr(dst + 2 * j * ktb), kreg + (size_t)ti * ktb, 2u * ktb, bar);
        for (int t = 0; t < 2; ++t)
          bulk_g2s(smem_addr(dst + 4 * ktb + (2 * j + t) * 128), vreg + (size_t)(ti + t) * vtb + VL::NORM, nb, bar);
      }
    } else {
      mbar_arrive_expect_tx(bar, (uint32_t)npairs * 2u * vtb);
      for (int j = 0; j < npairs; ++j)
        bulk_g2s(smem_addr(dst + 2 * j * vtb), vreg + (size_t)pair_index(tile0 + 2 * j) * vtb, 2u * vtb, bar);
    }
  };
  auto fail = [&]() {
    s_fail = 1;
    atomicOr(p.err, 1);
  };
  auto wait_fill = [&](int f) {
    const uint32_t bar = smem_addr(&fill_bar[(unsigned)f % kStagesT]), par = ((unsigned)f / kStagesT) & 1u;
    if (!mbar_try(bar, par) && !mbar_wait(bar, par, p.wait_limit)) fail();
  };
  auto wait_mma = [&](int g) {  // MMA group g (and everything issued before it) has completed
    const uint32_t bar = smem_addr(&mma_bar[g & 1]), par = ((unsigned)g >> 1) & 1u;
    if (!mbar_try(bar, par) && !mbar_wait(bar, par, p.wait_limit)) fail();
    tc::fence_after();
  };
  if (tid == 0)
#pragma unroll
    for (int f = 0; f < kStagesT - 1; ++f) issue(f);
  if (early) {
    grid_dep_wait();
    len = __ldcg(p.lens + b);
    t_end = min(len, t_begin + p.chunk);
    n_iter = t_end > t_begin ? (t_end - t_begin + kTokT - 1) / kTokT : 0;
    n_fill = 2 * n_iter;
  }
  if (p.debug_unset_wait && !mbar_wait(smem_addr(&fill_bar[kStagesT]), 0u, p.wait_limit)) fail();
  if (!p.cache_after_wait) grid_dep_wait();  // the prep area is the predecessor's output

  // ---- B_k: query digits of every plane in the octet words' byte order. K index 4x + i is byte i
  // of word x = 8t + 2m + hh, i.e. coordinate 32m + 16hh + 4t + i; row n = 2 h + digit.
  const int npiece = p.hsplit, gp = G / npiece;  // prep pieces of gp heads
  if (KV) {  // KIVI: the query itself; its digits are rebuilt per key group below
    for (int idx = tid; idx < G * kHeadDim; idx += kThreadsT)
      qsm[idx] = load_q(p.q, ((size_t)b * p.Hq + h_first + idx / kHeadDim) * kHeadDim + idx % kHeadDim, p.bf16) *
                 p.logit_scale;
    for (int idx = tid; idx < C::BK / 4; idx += kThreadsT) reinterpret_cast<uint32_t*>(bk)[idx] = 0u;
  }
  for (int idx = tid; idx < (KV ? 0 : KP * kKN * 32); idx += kThreadsT) {
    const int P = idx / (kKN * 32), n = (idx / 32) % kKN, x = idx % 32;
    uint32_t v = 0u;
    if (n < 2 * G) {
      const int h = n >> 1, d = n & 1, pc = h / gp, hp = h % gp;
      const unsigned char* area = p.qprep + (pair * npiece + pc) * p.qprep_stride;
      const int c0 = 32 * ((x >> 1) & 3) + 16 * (x & 1) + 4 * (x >> 3);
      v = __ldcg(reinterpret_cast<const uint32_t*>(area + ((P * gp + hp) * 2 + d) * 128 + c0));
    }
    *reinterpret_cast<uint32_t*>(bk + P * (kKN * 128) + core_off(n, 4 * x, 8)) = v;
  }
  for (int idx = tid; idx < 2 * C::BV / 4; idx += kThreadsT) reinterpret_cast<uint32_t*>(bv)[idx] = 0u;
  // head constants of this thread's heads (warp half hf: heads hf * GH ..)
  float hs[GH], hc[GH], hsz[GH], hcz[GH];
#pragma unroll
  for (int i = 0; i < GH; ++i) {
    hs[i] = hc[i] = hsz[i] = hcz[i] = 0.f;
    if (KV) continue;
    const int h = min(hf * GH + i, G - 1), pc = h / gp, hp = h % gp;
    const float* hconst =
        reinterpret_cast<const float*>(p.qprep + (pair * npiece + pc) * p.qprep_stride + KP * gp * 2 * 128);
    hs[i] = __ldcg(hconst + hp * 4 + 0);
    hc[i] = __ldcg(hconst + hp * 4 + 1);
    hsz[i] = __ldcg(hconst + hp * 4 + 2);
    hcz[i] = __ldcg(hconst + hp * 4 + 3);
  }
  fence_proxy_async();  // B_k and the zeroed B_v are read by the tensor cores
  __syncthreads();

  // key rows: token 32 qtr + lane of an iteration = tile qtr, slot lane, octet lane / 8, bit lane % 8
  const int oct = lane >> 3, jbit = lane & 7;
  const uint32_t kmask = 0x01010101u << jbit;
  const float rowf = -128.f / (float)(1 << jbit);  // u8 operand 2^j; head scales are in units of -128
  constexpr uint32_t kIdK = tc::idesc_i8(0, 1, 128, kKN);  // u8 key bits x s8 query digits
  constexpr uint32_t kIdV = tc::idesc_i8(0, 0, 128, NK0);  // u8 value bits x u8 weight digits
  float mrow[GH];
#pragma unroll
  for (int i = 0; i < GH; ++i) mrow[i] = -INFINITY;
  float wmax = 0.f, wmaxz = 0.f;
  float nk_prev = 0.f, gk_prev = 0.f;  // this thread's token row: key norm and residual norm

  // expansion of the planes of this warp half (plane P goes to half P % 2) into A buffer `abuf`
  auto expand = [&](const unsigned char* rowbase, int abuf, int nplanes, int walsh, int bits, int sketch_off,
                    uint32_t mask, int plane_stride) {
    for (int P = hf; P < nplanes; P += 2) {
      uint32_t r[32];
      auto load = [&](int off, uint32_t (&w)[32]) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(rowbase + off + c * plane_stride);
          w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
        }
      };
      if (P >= walsh) {
        load(sketch_off, r);
      } else if (bits == 3 && P == 3) {  // parity plane b0 ^ b1 ^ b2
        uint32_t t1[32];
        load(0, r);
        load(kTile * 16, t1);
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] ^= t1[c];
        load(2 * kTile * 16, t1);
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] ^= t1[c];
      } else {
        load(P * kTile * 16, r);
      }
#pragma unroll
      for (int c = 0; c < 32; ++c) r[c] &= mask;
      tc::tmem_st32(trow + C::COL_A + abuf * C::APL * 32 + P * 32, r);
    }
  };

  // logits of pass-1 iteration i from its accumulators (D_k buffer i & 1): this thread's token row
  auto key_epilogue = [&](int i) {
    wait_mma(i);
    uint32_t dm[8], dz[8];
    const uint32_t col = C::COL_DK + (i & 1) * 2 * kKN + 2 * hf * GH;
    tc::tmem_ld8(trow + col, dm);
    if (KQ) tc::tmem_ld8(trow + col + kKN, dz);
    tc::wait_ld();
    tc::fence_before();
    const int tok = i * kTokT + 32 * qtr + lane;  // chunk-relative
    const bool valid = t_begin + tok < t_end;
#pragma unroll
    for (int j = 0; j < GH; ++j) {
      const int h = hf * GH + j;
      const int c0 = (int)dm[2 * j], c1 = (int)dm[2 * j + 1];
      // hi * 256 + lo: exact in int32 up to 2 Walsh planes, else in fp32
      const float cc = KB <= 2 ? (float)(c0 * 256 + c1) : fmaf((float)c0, 256.f, (float)c1);
      if (KV) {  // KIVI: this group's digit scale and zero-point offset; no per-token norm
        const int hh = min(h, G - 1);
        const float lk = fmaf(hsk[(i & 1) * G + hh] * rowf, cc, hck[(i & 1) * G + hh]);
        const float lgk = valid ? lk : -INFINITY;
        if (h < G) {
          lgs[h * lgst + tok] = lgk;
          mrow[j] = fmaxf(mrow[j], lgk);
        }
        continue;
      }
      float l = fmaf(hs[j] * rowf, cc, hc[j]);
      if (KQ) {
        const int z0 = (int)dz[2 * j], z1 = (int)dz[2 * j + 1];
        l = fmaf(gk_prev, fmaf(hsz[j] * rowf, (float)(z0 * 256 + z1), hcz[j]), l);
      }
      const float lg = valid ? nk_prev * l : -INFINITY;
      if (h < G) {
        lgs[h * lgst + tok] = lg;
        mrow[j] = fmaxf(mrow[j], lg);
      }
    }
  };

  // ================= pass 1: logits of the whole chunk into lgs
  for (int it = 0; it < n_iter; ++it) {
    const int abuf = it % C::NBUF;
    if (C::NBUF == 1 && it > 0) wait_mma(it - 1);
    wait_fill(it);
    const unsigned char* kt = stages + ((unsigned)it % kStagesT) * C::STAGE;
    // this thread's token row: tile qtr, octet `oct` (words of every plane at stride 512)
    const unsigned char* krow = kt + qtr * ktb + oct * 128;
    if (KV) {
      // KIVI: the query digits of this key group, B_P[j] = 2^P q_j s_j (codes b0 + 2 b1), 16-bit
      // integers relative to the head's largest |2 q_j s_j|, into buffer it & 1; the head's offset
      // sum_j q_j z_j. Thread: coordinate j = tid % 128, heads tid / 128, + 2, ..
      const __half* st = reinterpret_cast<const __half*>(kt + 4 * ktb + kNormBlockT);
      const int j = tid & (kHeadDim - 1), h0 = tid >> 7;
      const float sj = __half2float(st[j]), zj = __half2float(st[kHeadDim + j]);
      constexpr int HT = (G + 1) / 2;
      float vq[HT];
#pragma unroll
      for (int u = 0; u < HT; ++u) {
        const int h = h0 + 2 * u;
        float a = 0.f, c = 0.f;
        vq[u] = 0.f;
        if (h < G) {
          vq[u] = qsm[h * kHeadDim + j] * sj;
          a = fabsf(vq[u]);
          c = qsm[h * kHeadDim + j] * zj;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
          c += __shfl_xor_sync(0xffffffffu, c, o);
        }
        if (lane == 0 && h < G) {
          kred[warp * G + h] = a;
          kred[8 * G + warp * G + h] = c;
        }
      }
      __syncthreads();
      if (tid < G) {  // head tid: warps 4 (tid & 1) .. +3 covered its coordinates
        const int w0 = 4 * (tid & 1);
        float a = 0.f, c = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          a = fmaxf(a, kred[(w0 + w) * G + tid]);
          c += kred[8 * G + (w0 + w) * G + tid];
        }
        const float vmax = 2.f * a;
        hsk[(it & 1) * G + tid] = (vmax > 0.f ? vmax : 1.f) / ((float)kQRange * -128.f);
        hck[(it & 1) * G + tid] = c;
        kred[16 * G + tid] = (float)kQRange / (vmax > 0.f ? vmax : 1.f);
      }
      __syncthreads();
      // K index of coordinate j = 32 m + 16 hh + 4 t + i: 4 (8 t + 2 m + hh) + i
      const int kidx = 4 * (8 * ((j >> 2) & 3) + 2 * (j >> 5) + ((j >> 4) & 1)) + (j & 3);
      unsigned char* bkb = bk + (it & 1) * (KP * kKN * 128);
#pragma unroll
      for (int u = 0; u < HT; ++u) {
        const int h = h0 + 2 * u;
        if (h >= G) continue;
        const float qs = kred[16 * G + h];
#pragma unroll
        for (int P = 0; P < 2; ++P) {
          const int q = __float2int_rn((float)(1 << P) * vq[u] * qs);
          const int hi = (q + 128) >> 8, lo = q - 256 * hi;
          bkb[P * (kKN * 128) + core_off(2 * h, kidx, 8)] = (unsigned char)(hi & 0xFF);
          bkb[P * (kKN * 128) + core_off(2 * h + 1, kidx, 8)] = (unsigned char)(lo & 0xFF);
        }
      }
      fence_proxy_async();  // the digits are read by the tensor cores after the barrier below
    }
    expand(krow, abuf, KP, KWP, KB, KL::SKETCH, kmask, 16);
    const float nk = __half2float(*reinterpret_cast<const __half*>(kt + qtr * ktb + KL::NORM + lane * 2));
    const float gk = KQ ? __half2float(*reinterpret_cast<const __half*>(kt + qtr * ktb + KL::GAMMA + lane * 2)) : 0.f;
    if (tid < kTokT && t_begin + it * kTokT + tid < t_end) {  // largest value weight of each kind
      const unsigned char* nb = kt + 4 * ktb + (tid / kTile) * 128 + (tid % kTile) * 2;
      const float w = __half2float(*reinterpret_cast<const __half*>(nb)) * (KV ? 1.f : kInvSqrtD);
      wmax = fmaxf(wmax, w);
      if (VQ) wmaxz = fmaxf(wmaxz, w * (__half2float(*reinterpret_cast<const __half*>(nb + 64)) * (kSqrtHalfPi / (float)p.v.m)));
    }
    tc::wait_st();
    tc::fence_before();
    __syncthreads();  // A complete; the stage is free for its refill
    if (tid == 0) {
      tc::fence_after();
      const uint32_t a0 = tmem + C::COL_A + abuf * C::APL * 32;
      const uint32_t dk = tmem + C::COL_DK + (it & 1) * 2 * kKN;
      const uint32_t bk0 = smem_addr(bk) + (KV ? (it & 1) * (KP * kKN * 128) : 0);
#pragma unroll
      for (int P = 0; P < KP; ++P) {
        const bool sk = KQ && P == KP - 1;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::umma_i8_ta(sk ? dk + kKN : dk, a0 + P * 32 + kk * 8,
                         tc::smem_desc(bk0 + P * (kKN * 128) + 2 * kk * 128, 128, 8 * 128), kIdK,
                         (sk ? kk > 0 : (P > 0 || kk > 0)) ? 1u : 0u);
      }
      tc::commit(smem_addr(&mma_bar[it & 1]));
      issue(it + kStagesT - 1);
    }
    if (it > 0) key_epilogue(it - 1);
    nk_prev = nk;
    gk_prev = gk;
  }
  if (n_iter > 0) key_epilogue(n_iter - 1);

  // chunk maxima per head, and the weight scales
  float* hmax = red;                // [8 warps][G]
  float* wred = red + 8 * G;        // [2][8]
  float* tsum = wred + 16;          // [3][threads]
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    float mx = mrow[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0 && hf * GH + j < G) hmax[warp * G + hf * GH + j] = mx;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
    wmaxz = fmaxf(wmaxz, __shfl_xor_sync(0xffffffffu, wmaxz, o));
  }
  if (lane == 0) { wred[warp] = wmax; wred[8 + warp] = wmaxz; }
  __syncthreads();
  float wm = 0.f, wmz = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) { wm = fmaxf(wm, wred[w]); wmz = fmaxf(wmz, wred[8 + w]); }
  const float wsc = wm > 0.f ? exp2f(floorf(log2f(kWRange / wm)) - 1.f) : 1.f;
  const float wscz = wmz > 0.f ? exp2f(floorf(log2f(kWRange / wmz)) - 1.f) : 1.f;
  const float vkappa = VQ ? kSqrtHalfPi / (float)p.v.m : 0.f;

  // ================= pass 2: weight digits, value contractions into D_v
  const bool has_task = tid < C::NTASK;
  const int task_h = min(tid / (kTokT / TPT), G - 1), task_T = TPT * (tid % (kTokT / TPT));
  float task_m = -INFINITY;
  if (has_task)
    for (int w = 0; w < 8; ++w)
      if ((w >> 2) * GH <= task_h && task_h < (w >> 2) * GH + GH) task_m = fmaxf(task_m, hmax[w * G + task_h]);
  float task_l = 0.f, task_zs = 0.f;  // task_zs (KIVI): sum of p_t z_t
  uint32_t task_wc = 0, task_wz = 0;
  // value rows: coordinate 32 qtr + lane = byte lane (4 qtr + lane / 8), bit lane % 8
  const int vlane = 4 * qtr + (lane >> 3);
  const uint32_t vmask = 0x01010101u << jbit;

  for (int it = 0; it < n_iter; ++it) {
    const int g = n_iter + it;  // MMA group number
    const int abuf = g % C::NBUF, bbuf = it & 1;
    // A buffer g % NBUF and B_v buffer it & 1 were last read by MMA group g - NBUF (NBUF = 1: the
    // group before, which completes after the one before it)
    if (it >= C::NBUF) wait_mma(g - C::NBUF);
    wait_fill(g);
    const unsigned char* vt = stages + ((unsigned)g % kStagesT) * C::STAGE;
    // weight digits of this iteration: p = 2^(l - m), both kinds, rounded by adding 2^23
    if (has_task) {
      const int tok0 = it * kTokT;
      unsigned char* bvb = bv + bbuf * C::BV;
      uint32_t bc[TPT], bz[TPT];
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < TPT; ++e) {
        const int T = task_T + e;
        const bool ok = t_begin + tok0 + T < t_end;
        const float lv = lgs[task_h * lgst + tok0 + T];
        const unsigned char* vtile = vt + (T / kTile) * vtb;
        const float pe = ok ? ex2(lv - task_m) : 0.f;
        psum += pe;
        const float nrm = ok ? __half2float(*reinterpret_cast<const __half*>(vtile + VL::NORM + (T % kTile) * 2)) : 0.f;
        bc[e] = __float_as_uint(fmaf(pe, nrm * ((KV ? 1.f : kInvSqrtD) * wsc), kRoundBias));
        task_wc += bc[e] - 0x4B000000u;
        if (KV && ok) task_zs = fmaf(pe, __half2float(*reinterpret_cast<const __half*>(vtile + VL::GAMMA + (T % kTile) * 2)), task_zs);
        if (VQ) {
          const float gz = ok ? __half2float(*reinterpret_cast<const __half*>(vtile + VL::GAMMA + (T % kTile) * 2)) : 0.f;
          bz[e] = __float_as_uint(fmaf(pe, nrm * gz * (kInvSqrtD * wscz * vkappa), kRoundBias));
          task_wz += bz[e] - 0x4B000000u;
        }
      }
      task_l += psum;
#pragma unroll
      for (int kind = 0; kind < C::NKIND; ++kind) {
        const uint32_t* bw = kind ? bz : bc;
#pragma unroll
        for (int d = 0; d < 3; ++d) {  // digit d = byte 2 - d of the rounded floats
          const int n = kind * NK0 + 3 * task_h + d;
          unsigned char* dst = bvb + core_off(n, task_T, kTokT / 16);
          if (TPT == 4) {
            const uint32_t lo = __byte_perm(bw[0], bw[TPT > 1 ? 1 : 0], (2 - d) | ((6 - d) << 4));
            const uint32_t hi = __byte_perm(bw[TPT > 2 ? 2 : 0], bw[TPT > 3 ? 3 : 0], (2 - d) | ((6 - d) << 4));
            *reinterpret_cast<uint32_t*>(dst) = (lo & 0xFFFFu) | (hi << 16);
          } else if (TPT == 2) {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)__byte_perm(bw[0], bw[TPT > 1 ? 1 : 0], (2 - d) | ((6 - d) << 4));
          } else {
            *dst = (unsigned char)(bw[0] >> (8 * (2 - d)));
          }
        }
      }
    }
    // value bits of this thread's coordinate row for the iteration's four tiles: byte lane `vlane`
    // of each tile is 32 contiguous bytes (one token each)
    for (int P = hf; P < VP; P += 2) {
      uint32_t r[32];
      auto load = [&](int off, uint32_t (&w)[32]) {
#pragma unroll
        for (int t4 = 0; t4 < 4; ++t4) {
          const unsigned char* src = vt + t4 * vtb + off + vlane * kTile;
          const uint4 v0 = *reinterpret_cast<const uint4*>(src), v1 = *reinterpret_cast<const uint4*>(src + 16);
          w[8 * t4] = v0.x; w[8 * t4 + 1] = v0.y; w[8 * t4 + 2] = v0.z; w[8 * t4 + 3] = v0.w;
          w[8 * t4 + 4] = v1.x; w[8 * t4 + 5] = v1.y; w[8 * t4 + 6] = v1.z; w[8 * t4 + 7] = v1.w;
        }
      };
      if (P >= VWP) {
        load(VL::SKETCH, r);
      } else if (VB == 3 && P == 3) {
        uint32_t t1[32];
        load(0, r);
        load(kTile * 16, t1);
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] ^= t1[c];
        load(2 * kTile * 16, t1);
#pragma unroll
        for (int c = 0; c < 32; ++c) r[c] ^= t1[c];
      } else {
        load(P * kTile * 16, r);
      }
      // tiles past the end of the chunk's data were not filled: their tokens have zero weights,
      // but their bytes are whatever the stage held, which is harmless (0 x anything = 0)
#pragma unroll
      for (int c = 0; c < 32; ++c) r[c] &= vmask;
      tc::tmem_st32(trow + C::COL_A + abuf * C::APL * 32 + P * 32, r);
    }
    tc::wait_st();
    tc::fence_before();
    fence_proxy_async();  // the weight digits are read by the tensor cores
    __syncthreads();
    if (tid == 0) {
      tc::fence_after();
      const uint32_t a0 = tmem + C::COL_A + abuf * C::APL * 32;
      const uint32_t bv0 = smem_addr(bv + bbuf * C::BV);
#pragma unroll
      for (int P = 0; P < VP; ++P) {
        const int kind = (VQ && P == VP - 1) ? 1 : 0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc::umma_i8_ta(tmem + C::COL_DV + P * NK0, a0 + P * 32 + kk * 8,
                         tc::smem_desc(bv0 + ((kind * NK0 / 8) * 8 + 2 * kk) * 128, 128, 8 * 128), kIdV,
                         (it > 0 || kk > 0) ? 1u : 0u);
      }
      tc::commit(smem_addr(&mma_bar[g & 1]));
      issue(g + kStagesT - 1);
    }
  }
  if (n_iter > 0) wait_mma(2 * n_iter - 1);

  grid_dep_launch();  // let the split reduce be scheduled; it waits for this grid to finish
  // ================= finish: per-head sums of p and of the weights, then this thread's rows
  // After a wait that gave up, thread 0 waits once more (bounded) for the last fill of each stage.
  if (tid == 0 && s_fail)
    for (int f = max(0, n_fill - kStagesT); f < n_fill; ++f)
      mbar_wait(smem_addr(&fill_bar[(unsigned)f % kStagesT]), ((unsigned)f / kStagesT) & 1u, p.wait_limit);
  tsum[tid] = task_l;
  tsum[kThreadsT + tid] = (float)task_wc;
  tsum[2 * kThreadsT + tid] = (float)task_wz;
  tsum[3 * kThreadsT + tid] = task_zs;
  __syncthreads();
  float* hsum = hmax;  // [4][G] (the maxima are folded into registers first)
  float mfin[GH];
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    const int h = min(hf * GH + j, G - 1);
    float mx = -INFINITY;
    for (int w = 0; w < 8; ++w)
      if ((w >> 2) * GH <= h && h < (w >> 2) * GH + GH) mx = fmaxf(mx, hmax[w * G + h]);
    mfin[j] = mx;
  }
  __syncthreads();
  if (tid < 4 * G) {
    const int what = tid / G, h = tid % G;
    float s2 = 0.f;
    for (int q = 0; q < kTokT / TPT; ++q) s2 += tsum[what * kThreadsT + h * (kTokT / TPT) + q];
    hsum[what * G + h] = s2;
  }
  __syncthreads();

  float va[4];
  walsh_coeffs(VB, p.v.cent, va);
  float vasum = 0.f;
#pragma unroll
  for (int P = 0; P < VWP; ++P) vasum += va[P];
  if (KV) {  // KIVI codes b0 + 2 b1: plane coefficients 1 and 2, no Walsh offset
    va[0] = 0.5f;
    va[1] = 1.f;
    vasum = 0.f;
  }
  const int j_c = 32 * qtr + lane;                  // this thread's coordinate row
  const float rowpos = 1.f / (float)(1 << jbit);    // row value 2^p (u8)
  const float rowinv = rowpos / wsc, rowinvz = rowpos / wscz;
  float o[GH], z[GH];
#pragma unroll
  for (int j = 0; j < GH; ++j) { o[j] = 0.f; z[j] = 0.f; }
  if (n_iter > 0) {
#pragma unroll
    for (int P = 0; P < VP; ++P) {
      const bool sk = VQ && P == VP - 1;
      uint32_t r[NK0 > 16 ? 32 : 16];
      if constexpr (NK0 > 16) {
        tc::tmem_ld32(trow + C::COL_DV + P * NK0, r);
      } else {
        tc::tmem_ld16(trow + C::COL_DV + P * NK0, r);
      }
      tc::wait_ld();
#pragma unroll
      for (int j = 0; j < GH; ++j) {
        const int h = min(hf * GH + j, G - 1);
        const float rr = fmaf((float)r[3 * h], 65536.f, fmaf((float)r[3 * h + 1], 256.f, (float)r[3 * h + 2]));
        if (sk) z[j] = 2.f * rr * rowinvz;
        else o[j] = fmaf(2.f * va[min(P, 3)], rr * rowinv, o[j]);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < GH; ++j) {
    const int h = hf * GH + j;
    if (h < G) {
      float* dst = p.part + (((size_t)b * p.Hq + h_first + h) * p.splits + split) * p.part_stride;
      dst[2 + j_c] = KV ? o[j] + hsum[3 * G + h] : o[j] - vasum * (hsum[G + h] / wsc);
      if (VQ) dst[2 + kHeadDim + j_c] = z[j] - hsum[2 * G + h] / wscz;
      if (lane == 0 && qtr == 0) {
        dst[0] = mfin[j];
        dst[1] = hsum[h];
      }
    }
  }

  // ---- teardown: after a wait that gave up, wait once more (bounded) for the last MMAs
  if (tid == 0 && s_fail && n_iter > 0) mbar_wait(smem_addr(&mma_bar[(2 * n_iter - 1) & 1]),
                                                 ((unsigned)(2 * n_iter - 1) >> 1) & 1u, p.wait_limit);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::dealloc(tmem, kTmemColsT);
  }
}

template <int G, int KB, bool KQ, int VB, bool VQ, bool KV = false>
cudaError_t launch_tc(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  using C = TcCfg<G, KB, KQ, VB, VQ, KV>;
  if (!C::KL::matches(p.k) || !C::VL::matches(p.v)) return cudaErrorNotSupported;
  if (p.k.order != kOrderOctet || p.v.order != kOrderByteLane) return cudaErrorNotSupported;
  cudaError_t e = cudaSuccess;
  if (!KV && (e = launch_lm_query_prep(p, s, qp)) != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  const size_t smem = tc_smem_bytes<C>(G, p.chunk);
  auto kern = decode_lm_tc<G, KB, KQ, VB, VQ, KV>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, p.Hkv, p.B);
  cfg.blockDim = dim3(kThreadsT);
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
cudaError_t dispatch_tc(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  const int kb = p.k.bits, vb = p.v.bits;
  const bool kq = p.k.qjl, vq = p.v.qjl;
#define KVQ_TC_CASE(KB, KQ, VB, VQ) \
  if (kb == KB && kq == KQ && vb == VB && vq == VQ) return launch_tc<G, KB, KQ, VB, VQ>(p, s, ev_mid, qp);
  KVQ_TC_CASE(2, true, 2, true)
  KVQ_TC_CASE(3, true, 3, false)
  KVQ_TC_CASE(1, false, 1, false)
  KVQ_TC_CASE(2, true, 2, false)
  KVQ_TC_CASE(3, true, 3, true)
  KVQ_TC_CASE(2, false, 2, false)
  KVQ_TC_CASE(3, false, 3, false)
#undef KVQ_TC_CASE
  return cudaErrorNotSupported;
}

}  // namespace

bool tc_modes_supported(int group, int k_bits, int k_qjl, int v_bits, int v_qjl) {
  return (group == 1 || group == 2 || group == 4 || group == 8) &&
         mma_modes_supported(group, k_bits, k_qjl, v_bits, v_qjl);
}

int tc_chunk_max(int group) { return group > 4 ? 4096 : 8192; }

bool tc_decode_supported(const DecodeParams& p) {
  return tc_modes_supported(p.group, p.k.bits, p.k.qjl, p.v.bits, p.v.qjl) && p.k.order == kOrderOctet &&
         p.chunk % 64 == 0 && p.chunk <= tc_chunk_max(p.group) && p.qprep != nullptr &&
         p.hsplit == (p.group > 4 ? 2 : 1);
}

cudaError_t launch_decode_kivi_tc(const DecodeParams& p, cudaStream_t s) {
  if (p.chunk % kTokT) return cudaErrorNotSupported;  // iterations are whole key groups
  switch (p.group) {
    case 1: return launch_tc<1, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    case 2: return launch_tc<2, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    case 4: return launch_tc<4, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    case 8: return launch_tc<8, 2, false, 2, false, true>(p, s, nullptr, nullptr);
    default: return cudaErrorNotSupported;
  }
}

cudaError_t launch_decode_lm_tc(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  switch (p.group) {
    case 1: return dispatch_tc<1>(p, s, ev_mid, qp);
    case 2: return dispatch_tc<2>(p, s, ev_mid, qp);
    case 4: return dispatch_tc<4>(p, s, ev_mid, qp);
    case 8: return dispatch_tc<8>(p, s, ev_mid, qp);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kvq
