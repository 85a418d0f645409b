// Warp-specialised split-K decode attention for LM / LM_QJL / SIGN1 caches on the 5th-generation
// tensor cores (tcgen05.mma kind::i8, accumulators in tensor memory).
//
// The computation and its integer formulation are those of the other LM decode kernels
// ("TurboQuant vs OSCAR vs EpiCache", section "Quantization frontiers: TurboQuant and OSCAR":
// logits from the Lloyd-Max centroids plus the unbiased QJL correction, softmax, values dequantised
// on the fly; Walsh planes, 16-bit query digits, 23-bit weight digits, two passes per chunk; see
// kvq_decode_tc.cu for the operand layouts). What differs is how the CTA's warps share the work:
// instead of every warp taking every step between CTA barriers, each warp has one role and the
// roles hand work to each other through mbarriers, so expansion, tensor-core products and
// epilogues of neighbouring iterations overlap.
//   * warps 12-13: the bulk copies of the cache tiles into the shared-memory stages, fill f by warp
//     12 + f % 2, each as soon as the stage's previous contents have been consumed. A copy
//     instruction holds its thread for about 140 ns whatever its size (1-16 KB), so a fill is as few
//     copies as the layout allows: its tiles in one copy (one per page of a paged cache), plus one
//     small copy per tile for the value norms that pass 1 needs;
//   * warps 14-15 (one thread each): the tcgen05.mma issue, pass 1 by alternate iterations and
//     pass 2 by alternate planes (one instruction takes an issuing thread about 50 cycles, and
//     threads issue in parallel), committing to the barriers of whoever waits;
//   * warps 0-7, expansion: key bits (pass 1) and value bits (pass 2) of the iteration's 128 tokens
//     expanded into one of the tensor-memory A buffers; warp w reaches lanes 32 (w % 4) .. + 31 and
//     takes half of the planes (w / 4);
//   * warps 8-11, epilogue: pass 1 reads each iteration's logit accumulators and writes the chunk's
//     logits; pass 2 turns logits and value norms into the weight digits (the B operand) of each
//     iteration; at the end they read the value accumulators and write the partials.
// A warp's 32 token rows are one octet of each of the iteration's four key tiles, which are staged
// contiguously as they lie in the cache. Every wait is bounded; after one
// gives up (bit 0 of the cache's status word) the CTA's later waits return at once, and the kernel
// still waits, bounded, for its own copies and products before it frees its tensor memory.
#include <algorithm>

#include <cuda_fp16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_lm_common.cuh"
#include "kvq_tcgen05.cuh"
#include "kvq_tiles.cuh"

// WsCfg members unused by the one configuration that falls back to the lockstep kernel
#pragma nv_diag_suppress 177

namespace kvq {
namespace {

using namespace lmc;

constexpr int kTokW = 128;                          // tokens per iteration (four cache tiles)
constexpr int kMaxStagesW = 12;                     // bulk-copy stages: as many as shared memory holds
constexpr int kSmemW = 227 * 1024;                  // dynamic shared memory of one CTA (at most)
constexpr int kNBV = 4;                             // weight-digit (B_v) buffers
constexpr int kExpW = 8;                            // expansion warps 0 .. 7
constexpr int kEpiW = 4;                            // epilogue warps 8 .. 11
constexpr int kProdW = kExpW + kEpiW;               // warps 12, 13: bulk copies
constexpr int kNProd = 2;
constexpr int kIssW = kProdW + kNProd;              // warps 14, 15: MMA issue (16 warps: 128 registers)
constexpr int kNIss = 2;
constexpr int kThreadsW = (kIssW + kNIss) * 32;
constexpr uint32_t kTmemColsW = 512;
constexpr int kKNW = 16;                            // key-phase N: 8 heads x 2 digits
constexpr int kEpiBar = 1;                          // named barrier of the 128 epilogue threads

template <int G, int KB, bool KQ, int VB, bool VQ>
struct WsCfg {
  static constexpr int KWP = Walsh<KB>::P, KP = KWP + (KQ ? 1 : 0);  // key planes (sketch last)
  static constexpr int VWP = Walsh<VB>::P, VP = VWP + (VQ ? 1 : 0);  // value planes (sketch last)
  static constexpr int NKIND = VQ ? 2 : 1;
  static constexpr int NK0 = ((3 * G + 15) / 16) * 16;  // value-phase N per kind: column 3 h + digit
  static constexpr int VN = NKIND * NK0;
  static constexpr int APL = KP > VP ? KP : VP;         // planes of one A buffer (32 columns each)
  // Tensor memory: NA A buffers, DKB key accumulators [main 16 | sketch 16], the value accumulators
  // [VP][NK0]; as many buffers as fit (A up to 8, key accumulators 4, else 2), so that expansion,
  // products and epilogues run several iterations apart
  static constexpr int DV = VP * NK0;
  static constexpr int DKB = (kTmemColsW - 4 * 2 * kKNW - DV) / (APL * 32) >= 2 ? 4 : 2;
  static constexpr int NA0 = ((int)kTmemColsW - DKB * 2 * kKNW - DV) / (APL * 32);
  static constexpr int NA = NA0 > 8 ? 8 : NA0;
  static constexpr uint32_t COL_A = 0;                  // buffer a at COL_A + a * APL * 32
  static constexpr uint32_t COL_DK = NA * APL * 32;
  static constexpr uint32_t COL_DV = COL_DK + DKB * 2 * kKNW;
  // two A buffers and every accumulator fit in the 512 columns (all but 8 heads with 3-bit + QJL
  // keys and values, which the lockstep kernel's single A buffer serves)
  static constexpr bool FITS = NA >= 2;
  using KL = TileLayout<KB, KQ>;
  using VL = TileLayout<VB, VQ>;
  static constexpr int KT = KL::BYTES;                        // staged key tile stride
  static constexpr int KNORM = 4 * KT;                        // value norms (+ gammas) of the four tiles
  static constexpr int KSTAGE = KNORM + 4 * 128;
  static constexpr int VSTAGE = 4 * VL::BYTES;
  static constexpr int STAGE = ((KSTAGE > VSTAGE ? KSTAGE : VSTAGE) + 127) / 128 * 128;
  static constexpr int BK = KP * kKNW * 128;                  // query digits, [KP][16 rows][128 K]
  static constexpr int BV = VN * kTokW;                       // one weight-digit buffer (kNBV of them)
  static constexpr int TPT = G;                               // tokens per weight task (128 tasks)
  static constexpr int CHUNK = G > 4 ? 4096 : 8192;           // largest chunk (the split plan's bound)
  static constexpr int LGS = 4 * G * ((CHUNK + kTokW - 1) / kTokW * kTokW + 8);
  static constexpr int FIXED = BK + kNBV * BV + LGS + 4 * (8 * G + 8 + 3 * kTokW + 3 * G) + 1024;
  static constexpr int NS0 = (kSmemW - FIXED) / STAGE;
  static constexpr int NS = NS0 > kMaxStagesW ? kMaxStagesW : NS0;  // stages
};

__host__ __device__ inline int ws_logit_stride(int chunk) { return (chunk + kTokW - 1) / kTokW * kTokW + 8; }

// Dynamic shared memory: stages | B_k | kNBV x B_v | logits [G][stride] | head constants | reductions.
template <class C>
size_t ws_smem_bytes(int G, int chunk) {
  return (size_t)C::NS * C::STAGE + C::BK + kNBV * C::BV +
         sizeof(float) * ((size_t)G * ws_logit_stride(chunk) + 4 * G + 4 * G + 8 + 3 * kTokW + 3 * G);
}

__device__ __forceinline__ int core_off_w(int n, int k, int kchunks) {
  return ((n >> 3) * kchunks + (k >> 4)) * 128 + (n & 7) * 16 + (k & 15);
}

__device__ __forceinline__ float half_at(const unsigned char* p) { return __half2float(*reinterpret_cast<const __half*>(p)); }

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

template <int G, int KB, bool KQ, int VB, bool VQ>
__global__ void __launch_bounds__(kThreadsW, 1) decode_lm_ws(const __grid_constant__ DecodeParams p) {
  using C = WsCfg<G, KB, KQ, VB, VQ>;
  using KL = typename C::KL;
  using VL = typename C::VL;
  constexpr int KP = C::KP, VP = C::VP, VWP = C::VWP, NK0 = C::NK0, TPT = C::TPT, NA = C::NA, DKB = C::DKB;
  constexpr int kStagesW = C::NS;
  static_assert(kStagesW >= 4, "stages");
  constexpr int vtb = VL::BYTES;
  extern __shared__ __align__(1024) unsigned char smem[];
  // barriers: stage full / consumed, A buffer full / free, key accumulator full / free, weight
  // digits full / free, value products done, one nothing completes (test entry). A ring of R uses
  // slot u % R and completes phase u / R of its barriers.
  enum {
    FULL = 0, EMPTY = FULL + kMaxStagesW, AF = EMPTY + kMaxStagesW, AE = AF + 8, DKF = AE + 8, DKE = DKF + 4,
    BVF = DKE + 4, BVE = BVF + kNBV, DVD = BVE + kNBV, UNSET = DVD + 1, NBAR = UNSET + 1
  };
  __shared__ __align__(8) uint64_t bars[NBAR];
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_fail;

  const int lgst = ws_logit_stride(p.chunk);
  unsigned char* stages = smem;
  unsigned char* bk = stages + kStagesW * C::STAGE;
  unsigned char* bv = bk + C::BK;
  float* lgs = reinterpret_cast<float*>(bv + kNBV * C::BV);
  float* hcon = lgs + G * lgst;  // [G][4]: head scale, offset, sketch scale, sketch offset
  float* red = hcon + 4 * G;     // epilogue reductions

  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t_begin = split * p.chunk;
  const size_t pair = (size_t)b * p.Hkv + hk;
  const int h_first = hk * p.group;
  const unsigned char* kreg = reinterpret_cast<const unsigned char*>(p.kreg);
  const unsigned char* vreg = reinterpret_cast<const unsigned char*>(p.vreg);
  auto bar = [&](int i) { return smem_addr(&bars[i]); };

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < kStagesW; ++s) {
      mbar_init(bar(FULL + s), 1);
      mbar_init(bar(EMPTY + s), kExpW + kEpiW);
    }
    for (int i = 0; i < NA; ++i) {
      mbar_init(bar(AF + i), kExpW);
      mbar_init(bar(AE + i), kNIss);
    }
    for (int i = 0; i < DKB; ++i) {
      mbar_init(bar(DKF + i), 1);
      mbar_init(bar(DKE + i), kEpiW);
    }
    for (int i = 0; i < kNBV; ++i) {
      mbar_init(bar(BVF + i), kEpiW);
      mbar_init(bar(BVE + i), kNIss);
    }
    mbar_init(bar(DVD), kNIss);
    mbar_init(bar(UNSET), 1);
    mbar_init_fence();
    s_fail = 0;
  }
  if (warp == 0) tc::alloc(smem_addr(&s_tmem), kTmemColsW);
  // The query prep area, and in a fused step the appended token and the lengths, are the
  // predecessor kernel's output: nothing is read before it has finished.
  grid_dep_wait();
  const int len = __ldcg(p.lens + b);
  const int t_end = min(len, t_begin + p.chunk);
  const int n_iter = t_end > t_begin ? (t_end - t_begin + kTokW - 1) / kTokW : 0;
  const int n_fill = 2 * n_iter;

  // ---- B_k: query digits of every plane in the octet words' byte order (K index 4x + i is byte i
  // of word x = 8t + 2m + hh, coordinate 32m + 16hh + 4t + i); row n = 2 h + digit
  const int npiece = p.hsplit, gp = G / npiece;  // prep pieces of gp heads
  for (int idx = tid; idx < KP * kKNW * 32; idx += kThreadsW) {
    const int P = idx / (kKNW * 32), n = (idx / 32) % kKNW, x = idx % 32;
    uint32_t v = 0u;
    if (n < 2 * G) {
      const int h = n >> 1, d = n & 1, pc = h / gp, hp = h % gp;
      const unsigned char* area = p.qprep + (pair * npiece + pc) * p.qprep_stride;
      const int c0 = 32 * ((x >> 1) & 3) + 16 * (x & 1) + 4 * (x >> 3);
      v = __ldcg(reinterpret_cast<const uint32_t*>(area + ((P * gp + hp) * 2 + d) * 128 + c0));
    }
    *reinterpret_cast<uint32_t*>(bk + P * (kKNW * 128) + core_off_w(n, 4 * x, 8)) = v;
  }
  for (int idx = tid; idx < 4 * G; idx += kThreadsW) {
    const int h = idx / 4, k = idx % 4, pc = h / gp, hp = h % gp;
    hcon[idx] = __ldcg(reinterpret_cast<const float*>(p.qprep + (pair * npiece + pc) * p.qprep_stride + KP * gp * 2 * 128) +
                       hp * 4 + k);
  }
  for (int idx = tid; idx < kNBV * C::BV / 4; idx += kThreadsW) reinterpret_cast<uint32_t*>(bv)[idx] = 0u;
  fence_proxy_async();  // B_k and the zeroed B_v are read by the tensor cores
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = s_tmem;
  if (p.debug_unset_wait && !mbar_wait(bar(UNSET), 0u, p.wait_limit)) atomicOr(p.err, 1);

  // bounded wait; once a wait of this CTA has given up, later ones return at once (results flagged)
  auto wait = [&](int i, uint32_t parity) {
    if (s_fail) return;
    if (!mbar_try(bar(i), parity) && !mbar_wait_spin(bar(i), parity, p.wait_limit)) {
      s_fail = 1;
      atomicOr(p.err, 1);
    }
  };

  if (warp >= kProdW && warp < kProdW + kNProd) {
    // ======================= bulk copies (one warp per fill)
    // Fill f < n_iter: the K tiles of pass-1 iteration f (lane 0: one copy; paged, lanes 0-1: one per
    // page) and their value norms (lanes 16-19); fill n_iter + i: the V tiles of pass-2 iteration i.
    // Tiles past the chunk's last token pair are not copied (their rows are masked or weighted zero).
    for (int f = warp - kProdW; f < n_fill; f += kNProd) {
      const int st = f % kStagesW;
      const uint32_t fb = bar(FULL + st);
      unsigned char* dst = stages + st * C::STAGE;
      const int it = f < n_iter ? f : f - n_iter;
      const int t0 = t_begin + it * kTokW;
      const int tile0 = (unsigned)t0 / kTile;
      const int ntiles = 2 * min(2, (t_end - t0 + 2 * kTile - 1) / (2 * kTile));
      constexpr uint32_t nb = VQ ? 128u : 64u;  // value norms (+ gammas, contiguous) per tile
      if (lane == 0) {
        if (f >= kStagesW) wait(EMPTY + st, ((unsigned)(f / kStagesW) - 1u) & 1u);
        fence_proxy_async();  // the stage's previous contents were read by the generic proxy
        mbar_arrive_expect_tx(fb, f < n_iter ? (uint32_t)ntiles * (KL::BYTES + nb) : (uint32_t)ntiles * vtb);
      }
      __syncwarp();
      if (f < n_iter) {
        if (!p.table) {
          if (lane == 0 && ntiles > 0) {
            const long ti = tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk, tile0, p.err);
            bulk_g2s(smem_addr(dst), kreg + (size_t)ti * KL::BYTES, (uint32_t)ntiles * KL::BYTES, fb);
          }
        } else if (lane < ntiles / 2) {
          const long ti = tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk,
                                          tile0 + 2 * lane, p.err);
          bulk_g2s(smem_addr(dst + 2 * lane * KL::BYTES), kreg + (size_t)ti * KL::BYTES, 2u * KL::BYTES, fb);
        }
        if (lane >= 16 && lane - 16 < ntiles) {
          const long ti = tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk,
                                          tile0 + lane - 16, p.err);
          bulk_g2s(smem_addr(dst + C::KNORM + (lane - 16) * 128), vreg + (size_t)ti * vtb + VL::NORM, nb, fb);
        }
      } else {
        if (!p.table) {
          if (lane == 0 && ntiles > 0) {
            const long ti = tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk, tile0, p.err);
            bulk_g2s(smem_addr(dst), vreg + (size_t)ti * vtb, (uint32_t)ntiles * vtb, fb);
          }
        } else if (lane < ntiles / 2) {
          const long ti = tile_index_read(p.table, p.pages_per_seq, p.n_pages, p.tiles_per_seq, p.Hkv, b, hk,
                                          tile0 + 2 * lane, p.err);
          bulk_g2s(smem_addr(dst + 2 * lane * vtb), vreg + (size_t)ti * vtb, 2u * vtb, fb);
        }
      }
      __syncwarp();
    }
  } else if (warp >= kIssW) {
    // ======================= MMA issue (lane 0 of each issuing warp)
    // A thread's tcgen05.mma instructions issue about one per 50 cycles, so two threads share them:
    // pass 1 by iteration (each iteration's logits have their own accumulator), pass 2 by plane
    // (each plane has its own value accumulator); a buffer is free once both have committed to it.
    const int j = warp - kIssW;
    if (lane == 0) {
      constexpr uint32_t kIdK = tc::idesc_i8(0, 1, 128, kKNW);  // u8 key bits x s8 query digits
      constexpr uint32_t kIdV = tc::idesc_i8(0, 0, 128, NK0);   // u8 value bits x u8 weight digits
      const uint32_t bk0 = smem_addr(bk);
      for (int i = j; i < n_iter; i += kNIss) {
        const int ab = i % NA, db = i % DKB;
        wait(AF + ab, ((unsigned)i / NA) & 1u);
        if (i >= DKB) wait(DKE + db, ((unsigned)i / DKB - 1u) & 1u);
        tc::fence_after();
        const uint32_t a0 = tmem + C::COL_A + ab * C::APL * 32;
        const uint32_t dk = tmem + C::COL_DK + db * 2 * kKNW;
#pragma unroll
        for (int P = 0; P < KP; ++P) {
          const bool sk = KQ && P == KP - 1;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::umma_i8_ta(sk ? dk + kKNW : dk, a0 + P * 32 + kk * 8,
                           tc::smem_desc(bk0 + P * (kKNW * 128) + 2 * kk * 128, 128, 8 * 128), kIdK,
                           (sk ? kk > 0 : (P > 0 || kk > 0)) ? 1u : 0u);
        }
#pragma unroll
        for (int c = 0; c < kNIss; ++c) tc::commit(bar(AE + ab));
        tc::commit(bar(DKF + db));
      }
      for (int i = 0; i < n_iter; ++i) {
        const int g = n_iter + i, ab = g % NA, bb = i % kNBV;
        wait(AF + ab, ((unsigned)g / NA) & 1u);
        wait(BVF + bb, ((unsigned)i / kNBV) & 1u);
        tc::fence_after();
        const uint32_t a0 = tmem + C::COL_A + ab * C::APL * 32;
        const uint32_t bv0 = smem_addr(bv + bb * C::BV);
#pragma unroll
        for (int P = 0; P < VP; ++P) {
          if (P % kNIss != j) continue;
          const int kind = (VQ && P == VP - 1) ? 1 : 0;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc::umma_i8_ta(tmem + C::COL_DV + P * NK0, a0 + P * 32 + kk * 8,
                           tc::smem_desc(bv0 + ((kind * NK0 / 8) * 8 + 2 * kk) * 128, 128, 8 * 128), kIdV,
                           (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::commit(bar(AE + ab));
        tc::commit(bar(BVE + bb));
      }
      tc::commit(bar(DVD));  // arrives once every product issued above has completed
    }
  } else if (warp < kExpW) {
    // ======================= expansion: planes of this warp's rows into the A buffers
    const int qtr = warp & 3, hf = warp >> 2;
    const uint32_t trow = tmem + ((uint32_t)(32 * qtr) << 16);
    const int tt = lane >> 3, jbit = lane & 7;  // pass 1: octet qtr of tile tt, bit jbit
    // A plane's 32 words of this thread's row, masked to one bit per byte, into A buffer column col
    auto put = [&](uint32_t (&r)[32], uint32_t mask, uint32_t col) {
#pragma unroll
      for (int c = 0; c < 32; ++c) r[c] &= mask;
      tc::tmem_st32(trow + col, r);
    };
    // Planes of half hf: plane P for P = hf, hf + 2, ..; with 3-bit codes half 0 takes planes 0, 1
    // (and the sketch) and half 1 plane 2 and the parity plane b0 ^ b1 ^ b2 from the same loads.
    // All of a half's loads are issued before its first store (a tensor-memory store is a barrier
    // to the compiler, so loads after it would wait for it).
    auto expand = [&](auto load, int nwalsh, int bits, bool sketch, uint32_t mask, uint32_t col0) {
      uint32_t ra[32], rb[32];
      if (bits == 3) {
        if (hf == 0) {
          load(0, ra);
          load(1, rb);
          put(ra, mask, col0 + 0 * 32);
          put(rb, mask, col0 + 1 * 32);
          if (sketch) {
            load(-1, ra);
            put(ra, mask, col0 + nwalsh * 32);
          }
        } else {
          uint32_t rc[32];
          load(2, ra);
          load(0, rb);
          load(1, rc);
#pragma unroll
          for (int c = 0; c < 32; ++c) rc[c] ^= rb[c] ^ ra[c];
          put(ra, mask, col0 + 2 * 32);
          put(rc, mask, col0 + 3 * 32);
        }
      } else {
        const int np = nwalsh + (sketch ? 1 : 0);  // at most 3: planes hf and hf + 2
        if (hf < np) load(hf < nwalsh ? hf : -1, ra);
        if (hf + 2 < np) load(hf + 2 < nwalsh ? hf + 2 : -1, rb);
        if (hf < np) put(ra, mask, col0 + hf * 32);
        if (hf + 2 < np) put(rb, mask, col0 + (hf + 2) * 32);
      }
    };
    for (int i = 0; i < n_iter; ++i) {
      const int ab = i % NA, st = i % kStagesW;
      wait(FULL + st, ((unsigned)i / kStagesW) & 1u);
      if (i >= NA) wait(AE + ab, ((unsigned)i / NA - 1u) & 1u);
      tc::fence_after();
      const unsigned char* rowbase = stages + st * C::STAGE + tt * C::KT + qtr * 128;
      auto load = [&](int P, uint32_t (&w)[32]) {  // P = -1: the sketch words
        const unsigned char* src = rowbase + (P < 0 ? KL::SKETCH : KL::PLANES + P * (kTile * 16));
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 v = *reinterpret_cast<const uint4*>(src + c * 16);
          w[4 * c] = v.x; w[4 * c + 1] = v.y; w[4 * c + 2] = v.z; w[4 * c + 3] = v.w;
        }
      };
      expand(load, C::KWP, KB, KQ, 0x01010101u << jbit, C::COL_A + ab * C::APL * 32);
      __syncwarp();  // every lane's loads of the stage have been consumed by its stores
      if (lane == 0) mbar_arrive(bar(EMPTY + st));
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(AF + ab));
    }
    // pass 2: row 32 qtr + lane = byte lane 4 qtr + lane / 8, bit lane % 8 (coordinate 32 qtr + lane)
    const int vlane = 4 * qtr + (lane >> 3);
    for (int i = 0; i < n_iter; ++i) {
      const int g = n_iter + i, ab = g % NA, st = g % kStagesW;
      wait(FULL + st, ((unsigned)g / kStagesW) & 1u);
      if (g >= NA) wait(AE + ab, ((unsigned)g / NA - 1u) & 1u);
      tc::fence_after();
      const unsigned char* vt = stages + st * C::STAGE;
      auto load = [&](int P, uint32_t (&w)[32]) {  // byte lane vlane of the four tiles, 32 tokens each
        const int off = P < 0 ? VL::SKETCH : VL::PLANES + P * (kTile * 16);
#pragma unroll
        for (int t4 = 0; t4 < 4; ++t4) {
          const unsigned char* src = vt + t4 * vtb + off + vlane * kTile;
          const uint4 v0 = *reinterpret_cast<const uint4*>(src), v1 = *reinterpret_cast<const uint4*>(src + 16);
          w[8 * t4] = v0.x; w[8 * t4 + 1] = v0.y; w[8 * t4 + 2] = v0.z; w[8 * t4 + 3] = v0.w;
          w[8 * t4 + 4] = v1.x; w[8 * t4 + 5] = v1.y; w[8 * t4 + 6] = v1.z; w[8 * t4 + 7] = v1.w;
        }
      };
      // tiles past the chunk's data were not copied: their tokens have zero weights (0 x anything)
      expand(load, VWP, VB, VQ, 0x01010101u << jbit, C::COL_A + ab * C::APL * 32);
      __syncwarp();  // every lane's loads of the stage have been consumed by its stores
      if (lane == 0) mbar_arrive(bar(EMPTY + st));
      tc::wait_st();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(AF + ab));
    }
  } else {
    // ======================= epilogues (warps 8 .. 11, lane quarters 0 .. 3)
    const int qtr = warp - kExpW, et = tid - kExpW * 32;
    const uint32_t trow = tmem + ((uint32_t)(32 * qtr) << 16);
    const int tt = lane >> 3, jbit = lane & 7, slot = qtr * 8 + jbit;  // pass-1 row: tile tt, slot
    const float rowf = -128.f / (float)(1 << jbit);  // u8 operand 2^j; head scales in units of -128
    const float vkappa = VQ ? kSqrtHalfPi / (float)p.v.m : 0.f;
    float mrow[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mrow[h] = -INFINITY;
    float wmax = 0.f, wmaxz = 0.f;
    for (int i = 0; i < n_iter; ++i) {
      const int db = i % DKB, st = i % kStagesW;
      wait(FULL + st, ((unsigned)i / kStagesW) & 1u);
      // the stage's norms of this thread's token (key norm, residual norm, value norm and gamma),
      // then the stage is released: its refill does not wait for this iteration's products
      const unsigned char* kt = stages + st * C::STAGE;
      const int tok = i * kTokW + tt * kTile + slot;  // chunk-relative
      const bool valid = t_begin + tok < t_end;
      const float nk = half_at(kt + tt * C::KT + KL::NORM + slot * 2);
      const float gk = KQ ? half_at(kt + tt * C::KT + KL::GAMMA + slot * 2) : 0.f;
      const float wn = half_at(kt + C::KNORM + tt * 128 + slot * 2) * kInvSqrtD;
      const float wg = VQ ? half_at(kt + C::KNORM + tt * 128 + 64 + slot * 2) : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(EMPTY + st));
      wait(DKF + db, ((unsigned)i / DKB) & 1u);
      tc::fence_after();
      uint32_t dm[16], dz[16];
      tc::tmem_ld16(trow + C::COL_DK + db * 2 * kKNW, dm);
      if (KQ) tc::tmem_ld16(trow + C::COL_DK + db * 2 * kKNW + kKNW, dz);
      tc::wait_ld();
      tc::fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(DKE + db));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int c0 = (int)dm[2 * h], c1 = (int)dm[2 * h + 1];
        // hi * 256 + lo: exact in int32 up to 2 Walsh planes, else in fp32
        const float cc = KB <= 2 ? (float)(c0 * 256 + c1) : fmaf((float)c0, 256.f, (float)c1);
        float l = fmaf(hcon[4 * h] * rowf, cc, hcon[4 * h + 1]);
        if (KQ) {
          const int z0 = (int)dz[2 * h], z1 = (int)dz[2 * h + 1];
          l = fmaf(gk, fmaf(hcon[4 * h + 2] * rowf, (float)(z0 * 256 + z1), hcon[4 * h + 3]), l);
        }
        const float lg = valid ? nk * l : -INFINITY;
        lgs[h * lgst + tok] = lg;
        mrow[h] = fmaxf(mrow[h], lg);
      }
      if (valid) {  // the largest value weight of each kind (staged norms: [tile][64 B | 64 B gammas])
        wmax = fmaxf(wmax, wn);
        if (VQ) wmaxz = fmaxf(wmaxz, wn * (wg * vkappa));
      }
    }
    // chunk maxima per head and the weight scales, over the four epilogue warps
    float* hm = red;           // [4][G]
    float* wr = red + 4 * G;   // [2][4]
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = mrow[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) hm[qtr * G + h] = mx;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      wmax = fmaxf(wmax, __shfl_xor_sync(0xffffffffu, wmax, o));
      wmaxz = fmaxf(wmaxz, __shfl_xor_sync(0xffffffffu, wmaxz, o));
    }
    if (lane == 0) {
      wr[qtr] = wmax;
      wr[4 + qtr] = wmaxz;
    }
    named_sync(kEpiBar, kEpiW * 32);  // also orders every logit write before pass 2's reads
    float wm = 0.f, wmz = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      wm = fmaxf(wm, wr[w]);
      wmz = fmaxf(wmz, wr[4 + w]);
    }
    // integer weights below 2^23 (3 byte digits), each kind scaled by a power of two to its range
    const float wsc = wm > 0.f ? exp2f(floorf(log2f(kWRange / wm)) - 1.f) : 1.f;
    const float wscz = wmz > 0.f ? exp2f(floorf(log2f(kWRange / wmz)) - 1.f) : 1.f;
    // weight task: head task_h, tokens task_T .. task_T + TPT - 1 of each iteration
    const int task_h = et / (kTokW / TPT), task_T = TPT * (et % (kTokW / TPT));
    float task_m = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) task_m = fmaxf(task_m, hm[w * G + task_h]);
    float task_l = 0.f;
    uint32_t task_wc = 0, task_wz = 0;
    for (int i = 0; i < n_iter; ++i) {
      const int g = n_iter + i, st = g % kStagesW, bb = i % kNBV;
      wait(FULL + st, ((unsigned)g / kStagesW) & 1u);
      // the value norms (and gammas) of the task's tokens, then the stage is released
      const unsigned char* vt = stages + st * C::STAGE;
      float nrm[TPT], gzv[TPT];
#pragma unroll
      for (int e = 0; e < TPT; ++e) {
        const int T = task_T + e;
        const bool ok = t_begin + i * kTokW + T < t_end;
        const unsigned char* vtile = vt + (T / kTile) * vtb;
        nrm[e] = ok ? half_at(vtile + VL::NORM + (T % kTile) * 2) : 0.f;
        gzv[e] = (VQ && ok) ? half_at(vtile + VL::GAMMA + (T % kTile) * 2) : 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(EMPTY + st));
      if (i >= kNBV) wait(BVE + bb, ((unsigned)i / kNBV - 1u) & 1u);
      uint32_t bc[TPT], bz[TPT];
      float psum = 0.f;
#pragma unroll
      for (int e = 0; e < TPT; ++e) {
        const int T = task_T + e;
        const bool ok = t_begin + i * kTokW + T < t_end;
        const float pe = ok ? ex2(lgs[task_h * lgst + i * kTokW + T] - task_m) : 0.f;
        psum += pe;
        bc[e] = __float_as_uint(fmaf(pe, nrm[e] * (kInvSqrtD * wsc), kRoundBias));
        task_wc += bc[e] - 0x4B000000u;
        if (VQ) {
          bz[e] = __float_as_uint(fmaf(pe, nrm[e] * gzv[e] * (kInvSqrtD * wscz * vkappa), kRoundBias));
          task_wz += bz[e] - 0x4B000000u;
        }
      }
      task_l += psum;
      // digit d of the tokens' weights = byte 2 - d of the rounded floats, in row kind NK0 + 3 h + d;
      // the task's TPT tokens are TPT consecutive bytes of one core-matrix row
      unsigned char* bvb = bv + bb * C::BV;
#pragma unroll
      for (int kind = 0; kind < C::NKIND; ++kind) {
        const uint32_t* bw = kind ? bz : bc;
#pragma unroll
        for (int d = 0; d < 3; ++d) {
          unsigned char* dst = bvb + core_off_w(kind * NK0 + 3 * task_h + d, task_T, kTokW / 16);
          const int sh = 8 * (2 - d);
          if (TPT >= 4) {
#pragma unroll
            for (int q4 = 0; q4 < TPT / 4; ++q4) {
              uint32_t wv = 0u;
#pragma unroll
              for (int e = 0; e < 4; ++e) wv |= ((bw[4 * q4 + e] >> sh) & 0xFFu) << (8 * e);
              reinterpret_cast<uint32_t*>(dst)[q4] = wv;
            }
          } else {
#pragma unroll
            for (int e = 0; e < TPT; ++e) dst[e] = (unsigned char)(bw[e] >> sh);
          }
        }
      }
      fence_proxy_async();  // the digits are read by the tensor cores
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(BVF + bb));
    }
    grid_dep_launch();  // the split reduce may be scheduled; it waits for this grid to finish
    // ---- finish: value accumulators, per-head sums, this thread's coordinate row
    wait(DVD, 0u);
    tc::fence_after();
    float* tsum = wr + 8;              // [3][128]
    float* hsum = tsum + 3 * kTokW;    // [3][G]
    tsum[et] = task_l;
    tsum[kTokW + et] = (float)task_wc;
    tsum[2 * kTokW + et] = (float)task_wz;
    named_sync(kEpiBar, kEpiW * 32);
    if (et < 3 * G) {
      const int what = et / G, h = et % G;
      float s2 = 0.f;
      for (int q = 0; q < kTokW / TPT; ++q) s2 += tsum[what * kTokW + h * (kTokW / TPT) + q];
      hsum[et] = s2;
    }
    named_sync(kEpiBar, kEpiW * 32);
    float va[4];
    walsh_coeffs(VB, p.v.cent, va);
    float vasum = 0.f;
#pragma unroll
    for (int P = 0; P < VWP; ++P) vasum += va[P];
    const int j_c = 32 * qtr + lane;                 // this thread's coordinate row
    const float rowpos = 1.f / (float)(1 << jbit);   // row value 2^p (u8)
    const float rowinv = rowpos / wsc, rowinvz = rowpos / wscz;
    float o[G], z[G];
#pragma unroll
    for (int h = 0; h < G; ++h) { o[h] = 0.f; z[h] = 0.f; }
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
        for (int h = 0; h < G; ++h) {
          const float rr = fmaf((float)r[3 * h], 65536.f, fmaf((float)r[3 * h + 1], 256.f, (float)r[3 * h + 2]));
          if (sk) z[h] = 2.f * rr * rowinvz;
          else o[h] = fmaf(2.f * va[min(P, 3)], rr * rowinv, o[h]);
        }
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float* dst = p.part + (((size_t)b * p.Hq + h_first + h) * p.splits + split) * p.part_stride;
      dst[2 + j_c] = o[h] - vasum * (hsum[G + h] / wsc);
      if (VQ) dst[2 + kHeadDim + j_c] = z[h] - hsum[2 * G + h] / wscz;
      if (et == 0) {
        float mx = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) mx = fmaxf(mx, hm[w * G + h]);
        dst[0] = mx;
        dst[1] = hsum[h];
      }
    }
  }

  // ---- teardown: after a wait that gave up, the copying and issuing threads wait (bounded) for
  // their own last copies and products, so nothing lands after the memory is released
  if (warp == kProdW && lane == 0 && s_fail)
    for (int f = max(0, n_fill - kStagesW); f < n_fill; ++f)
      mbar_wait(bar(FULL + f % kStagesW), ((unsigned)f / kStagesW) & 1u, p.wait_limit);
  if (warp >= kIssW && lane == 0 && s_fail) mbar_wait(bar(DVD), 0u, p.wait_limit);
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::dealloc(tmem, kTmemColsW);
  }
}

template <int G, int KB, bool KQ, int VB, bool VQ>
cudaError_t launch_ws(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  using C = WsCfg<G, KB, KQ, VB, VQ>;
  if constexpr (!C::FITS) {
    return launch_decode_lm_tc(p, s, ev_mid, qp);
  } else {
  if (!C::KL::matches(p.k) || !C::VL::matches(p.v)) return cudaErrorNotSupported;
  if (p.k.order != kOrderOctet || p.v.order != kOrderByteLane) return cudaErrorNotSupported;
  cudaError_t e = launch_lm_query_prep(p, s, qp);
  if (e != cudaSuccess) return e;
  if (ev_mid && (e = cudaEventRecord(ev_mid, s)) != cudaSuccess) return e;
  const size_t smem = ws_smem_bytes<C>(G, p.chunk);
  auto kern = decode_lm_ws<G, KB, KQ, VB, VQ>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.splits, p.Hkv, p.B);
  cfg.blockDim = dim3(kThreadsW);
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
}

template <int G>
cudaError_t dispatch_ws(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  const int kb = p.k.bits, vb = p.v.bits;
  const bool kq = p.k.qjl, vq = p.v.qjl;
#define KVQ_WS_CASE(KB, KQ, VB, VQ) \
  if (kb == KB && kq == KQ && vb == VB && vq == VQ) return launch_ws<G, KB, KQ, VB, VQ>(p, s, ev_mid, qp);
  KVQ_WS_CASE(2, true, 2, true)
  KVQ_WS_CASE(3, true, 3, false)
  KVQ_WS_CASE(1, false, 1, false)
  KVQ_WS_CASE(2, true, 2, false)
  KVQ_WS_CASE(3, true, 3, true)
  KVQ_WS_CASE(2, false, 2, false)
  KVQ_WS_CASE(3, false, 3, false)
#undef KVQ_WS_CASE
  return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_decode_lm_ws(const DecodeParams& p, cudaStream_t s, cudaEvent_t ev_mid, const QuantizeParams* qp) {
  switch (p.group) {
    case 1: return dispatch_ws<1>(p, s, ev_mid, qp);
    case 2: return dispatch_ws<2>(p, s, ev_mid, qp);
    case 4: return dispatch_ws<4>(p, s, ev_mid, qp);
    case 8: return dispatch_ws<8>(p, s, ev_mid, qp);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace kvq
