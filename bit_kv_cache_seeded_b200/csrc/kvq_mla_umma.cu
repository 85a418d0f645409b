// 5th-generation tensor-core (tcgen05, accumulators in tensor memory) split-K decode attention
// over the FP4 MLA-style latent cache, for 64 query heads.
//
// "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2": one 512-dim latent per token is
// shared by all heads (section "CSA2") and stored as FP4 E2M1 with one scale per 16 channels
// (section "Numerics and hardware efficiency"; the scale is an E4M3 byte here). With the absorbed
// query q = [q_lat ; q_rope] each 64-token tile is two dense contractions:
//   S   = Q [64 heads x 576] . K^T [576 x 64 tokens]        (tcgen05.mma M=64, N=64, K=16 steps)
//   O^T += latent_hat^T [512 x 64 tokens] . P^T [64 x 64]   (tcgen05.mma M=128 x 4, N=64)
// latent_hat = E4M3 scale x E2M1 value is exact in f16; Q's latent part is scaled per head by a
// power of two into f16 range, its RoPE part stays bf16 (bf16 MMAs into the same accumulator).
//
// One CTA per SM (8 warps; warp w reaches tensor-memory lane quarter w % 4), per 64-token
// iteration:
//   1. every thread holds its share of the next tile's packed data in registers (loaded one tile
//      ahead) and dequantises it to f16, with the RoPE key, into the free one of two shared-memory
//      buffers in the canonical no-swizzle "core matrix" layout (8 rows x 16 B blocks) that both
//      MMAs read; this overlaps S of the current tile on the tensor cores;
//   2. S = Q K^T goes into tensor memory as two accumulators over halves of K (the latent's first
//      256 channels; the rest and the RoPE part), issued by lane 0 of warps 5 and 6, each committing
//      to the S barrier; one thread issues a tcgen05.mma only about every 50 cycles, so the 52
//      products of a tile are spread over four threads (O^T below on warps 4 and 7) that do no
//      softmax;
//   3. lanes 0..15 of warps 0..3 (the rows of S for an M=64 MMA) load and add their head's 64 logits,
//      update a lazily rescaled running maximum (rescale only when it grows by more than 8 in
//      log2 units), write P = 2^(l - m) (<= 256) as f16 in core-matrix layout;
//   4. if a head's maximum moved, every thread rescales that head's column of O^T in tensor
//      memory (load, multiply, store);
//   5. lane 0 of warps 4 and 7 issue O^T += latent^T P^T (two M-blocks each) and commit; warps 5 and
//      6 issue S of the next tile only after that (a named barrier of warps 4..7), so the tensor pipe
//      runs O^T first and the next iteration, which waits for O^T before it overwrites that latent
//      buffer, P or O, starts dequantising while S runs.
// Every mbarrier wait is bounded (the cache status word records a wait that gave up). Partials
// (m, l, o[512]) per (sequence, head, split) go to the workspace in the format of the other
// MLA kernels; the same reduce kernel finishes.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_async.cuh"
#include "kvq_internal.h"
#include "kvq_tcgen05.cuh"

namespace kvq {
namespace {

constexpr int kThreadsU = 256;          // 8 warps: warp w reaches tensor-memory lanes 32 (w % 4) ..
constexpr int kTokU = 64;               // tokens per iteration (two cache tiles)
constexpr int kLatU = 512, kRopeU = 64, kDqU = kLatU + kRopeU;
constexpr int kHeadsU = 64;
constexpr int kCore = 128;              // bytes of one core matrix (8 rows x 16 B)
constexpr float kLazyRescale = 8.f;     // rescale O only when the running max grows by more than this
constexpr uint32_t kTmemCols = 512;     // allocation: O^T in columns 0..255, S in 256..319 and 320..383
constexpr uint32_t kColO = 0, kColS = 256, kColS2 = 320;
constexpr int kWarpO = 4, kWarpO2 = 7, kWarpS = 5;  // O^T: lane 0 of warps 4, 7; S: of warps 5, 6
constexpr int kIssueBar = 2;                         // named barrier of warps 4..7: S after O^T

// Shared-memory layout (bytes). Q: [8 head groups][72 dim chunks] core matrices; LAT (x2): [8 token
// groups][64 dim chunks]; ROPE (x2): [8 token groups][8 dim chunks]; P: [8 head groups][8 token
// chunks]. The latent/RoPE buffers alternate between tiles.
constexpr int kOffQ = 0;
constexpr int kSizeQ = kHeadsU * kDqU * 2;              // 73728
constexpr int kOffLat = kOffQ + kSizeQ;                 // [2 buffers]
constexpr int kSizeLat = kTokU * kLatU * 2;             // 65536
constexpr int kOffRope = kOffLat + 2 * kSizeLat;        // [2 buffers]
constexpr int kSizeRope = kTokU * kRopeU * 2;           // 8192
constexpr int kOffP = kOffRope + 2 * kSizeRope;
constexpr int kSizeP = kHeadsU * kTokU * 2;             // 8192
constexpr int kSmemU = kOffP + kSizeP;                  // 229376

using tc::smem_desc;
using tc::idesc_f16;
using tc::umma_f16;
using tc::tmem_ld32;
using tc::tmem_st32;
__device__ __forceinline__ void umma_commit(uint32_t bar) { tc::commit(bar); }
__device__ __forceinline__ void tc_fence_before() { tc::fence_before(); }
__device__ __forceinline__ void tc_fence_after() { tc::fence_after(); }
__device__ __forceinline__ void tmem_wait_ld() { tc::wait_ld(); }
__device__ __forceinline__ void tmem_wait_st() { tc::wait_st(); }

// Two E2M1 codes (one byte, channel 2k in the low nibble) to f16x2 (channel 2k in the low half).
__device__ __forceinline__ uint32_t e2m1x2_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n .reg .b8 b;\n cvt.u8.u32 b, %1;\n cvt.rn.f16x2.e2m1x2 %0, b;\n}\n" : "=r"(r) : "r"(byte));
  return r;
}
// Two E4M3 bytes (low 16 bits) to f16x2.
__device__ __forceinline__ uint32_t e4m3x2_f16x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(r) : "h"((unsigned short)two));
  return r;
}
// 2^x with the hardware approximation (relative error ~2^-22; 2^-inf = +0).
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t hmul2u(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Byte offset of element (row, col) of a 16-bit matrix stored as core matrices with
// `chunks_per_row` 8-element column chunks per 8-row group: block (row/8, col/8) at
// ((row/8) * chunks_per_row + col/8) * 128, row % 8 at 16 B, col % 8 at 2 B.
__device__ __forceinline__ int core_off(int row, int col, int chunks_per_row) {
  return ((row >> 3) * chunks_per_row + (col >> 3)) * kCore + (row & 7) * 16 + (col & 7) * 2;
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) { tc::alloc(dst_smem, ncols); }
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) { tc::dealloc(taddr, ncols); }

// Packed data of one 64-token tile that one thread dequantises: token tid % 64, channels
// 128 (tid / 64) .. +127 (64 code bytes, 8 scale bytes) and two 16-byte RoPE chunks. Loaded straight
// from global memory into registers one tile ahead of its use.
struct TileRegs {
  uint4 codes[4];
  uint2 scales;
  uint4 rope[2];
};

__device__ __forceinline__ void load_tile(TileRegs& r, const unsigned char* base, const Fp4Layout& F, int tile_bytes,
                                          int t0, int count, int tid) {
  const int tok = tid & 63, quarter = tid >> 6, slot = tok & (kTile - 1);
  if (tok < count) {
    const unsigned char* ct = base + (size_t)((t0 >> 5) + (tok >> 5)) * tile_bytes;
#pragma unroll
    for (int j = 0; j < 4; ++j) {  // chunk order skewed by token: see dequant_tile
      const int c = (j + slot) & 3;
      r.codes[j] = *reinterpret_cast<const uint4*>(ct + F.off_codes + slot * (kLatU / 2) + quarter * 64 + c * 16);
    }
    r.scales = *reinterpret_cast<const uint2*>(ct + F.off_scales + slot * (kLatU / 16) + quarter * 8);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int dc = (quarter + 4 * k + tok) & 7;
      r.rope[k] = *reinterpret_cast<const uint4*>(ct + F.off_rope + slot * (kRopeU * 2) + dc * 16);
    }
  } else {  // zero codes and scales dequantise to zeros
#pragma unroll
    for (int j = 0; j < 4; ++j) r.codes[j] = make_uint4(0, 0, 0, 0);
    r.scales = make_uint2(0, 0);
    r.rope[0] = r.rope[1] = make_uint4(0, 0, 0, 0);
  }
}

// Dequantise one thread's share of a tile into core-matrix layout. The chunk order is skewed by
// token so that the 8 rows of each core matrix are written by 8 consecutive lanes (no conflicts).
__device__ __forceinline__ void dequant_tile(const TileRegs& r, unsigned char* lat, unsigned char* rope, int tid) {
  const int tok = tid & 63, quarter = tid >> 6, slot = tok & (kTile - 1);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = (j + slot) & 3;  // 32-channel chunk of this quarter: groups 2c, 2c+1
    const uint32_t sw = (c >> 1) ? r.scales.y : r.scales.x;
    const uint32_t s2 = e4m3x2_f16x2((sw >> (16 * (c & 1))) & 0xFFFFu);
    const uint32_t slo = s2 & 0xFFFFu, shi = s2 >> 16;
    const uint32_t bA = slo | (slo << 16), bB = shi | (shi << 16);
    const uint32_t w4[4] = {r.codes[j].x, r.codes[j].y, r.codes[j].z, r.codes[j].w};
    uint32_t out[16];
#pragma unroll
    for (int k = 0; k < 16; ++k)
      out[k] = hmul2u(e2m1x2_f16x2((w4[k >> 2] >> (8 * (k & 3))) & 0xFFu), k < 8 ? bA : bB);
    const int d0 = 128 * quarter + 32 * c;
#pragma unroll
    for (int v = 0; v < 4; ++v)
      *reinterpret_cast<uint4*>(lat + core_off(tok, d0 + 8 * v, kLatU / 8)) =
          make_uint4(out[4 * v], out[4 * v + 1], out[4 * v + 2], out[4 * v + 3]);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int dc = (quarter + 4 * k + tok) & 7;
    *reinterpret_cast<uint4*>(rope + core_off(tok, 8 * dc, kRopeU / 8)) = r.rope[k];
  }
}

__global__ void __launch_bounds__(kThreadsU, 1) decode_mla_umma(const __grid_constant__ MlaParams p) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ __align__(8) uint64_t bar_s;  // S = Q K^T done, both halves (their issuers' earlier MMAs too)
  __shared__ __align__(8) uint64_t bar_o;  // O^T += latent^T P^T done, both halves (earlier MMAs too)
  __shared__ uint32_t s_tmem;              // tensor-memory base address
  __shared__ float s_alpha[kHeadsU];       // per-head O rescale factor of this iteration
  __shared__ float s_hsc[kHeadsU];         // per-head power-of-two query scale
  __shared__ int s_fail;

  const Fp4Layout& F = p.fp4;
  const int tile_bytes = F.tile_bytes;
  unsigned char* sQ = smem + kOffQ;
  const int split = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int len = p.lens[b];
  const int t_begin = split * p.chunk;
  const int t_end = min(len, t_begin + p.chunk);
  const int n_iter = t_end > t_begin ? (t_end - t_begin + kTokU - 1) / kTokU : 0;
  const unsigned char* base = reinterpret_cast<const unsigned char*>(p.reg) + (size_t)b * p.tiles_per_seq * tile_bytes;
  auto tile_count = [&](int it) { return min(kTokU, t_end - (t_begin + it * kTokU)); };

  if (tid == 0) {
    mbar_init(smem_addr(&bar_s), 2);
    mbar_init(smem_addr(&bar_o), 2);
    mbar_init_fence();
    s_fail = 0;
  }
  if (warp == 0) tmem_alloc(smem_addr(&s_tmem), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t tmem_warp = tmem + ((uint32_t)(32 * (warp & 3)) << 16);  // this warp's lane quarter
  const int col_half = warp >> 2;  // O^T columns (heads) 32 col_half .. +31 for rescale and output
  auto wait_bar = [&](uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_addr(bar);
    if (!mbar_try(a, parity) && !mbar_wait(a, parity, p.wait_limit)) {
      s_fail = 1;
      atomicOr(p.err, 1);
    }
  };

  TileRegs regs;
  if (n_iter > 0) load_tile(regs, base, F, tile_bytes, t_begin, tile_count(0), tid);

  // ---- Q: per-head power-of-two scale into f16 range; latent part f16, RoPE part bf16, stored
  // as core matrices [8 head groups][72 dim chunks] (K-major A operand of S = Q K^T)
  const size_t qbase = (size_t)b * kHeadsU * kDqU;
  for (int h = warp; h < kHeadsU; h += kThreadsU / 32) {
    const void* qh = p.bf16 ? (const void*)(reinterpret_cast<const __nv_bfloat16*>(p.q) + qbase + (size_t)h * kDqU)
                            : (const void*)(reinterpret_cast<const float*>(p.q) + qbase + (size_t)h * kDqU);
    float mx = 0.f;
    for (int c = lane; c < kDqU; c += 32) {
      const float v = p.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(qh)[c])
                             : reinterpret_cast<const float*>(qh)[c];
      mx = fmaxf(mx, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float sc = mx > 0.f ? exp2f(ceilf(log2f(mx)) - 14.f) : 1.f;
    if (lane == 0) s_hsc[h] = sc;
    const float inv = 1.f / sc;
    for (int c = lane; c < kDqU; c += 32) {
      const float v = (p.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(qh)[c])
                              : reinterpret_cast<const float*>(qh)[c]) * inv;
      unsigned char* dst = sQ + core_off(h, c, kDqU / 8);
      if (c < kLatU) *reinterpret_cast<__half*>(dst) = __float2half_rn(v);
      else *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(v);
    }
  }
  // first tile into buffer 0, then fetch the second
  if (n_iter > 0) dequant_tile(regs, smem + kOffLat, smem + kOffRope, tid);
  if (n_iter > 1) load_tile(regs, base, F, tile_bytes, t_begin + kTokU, tile_count(1), tid);
  fence_proxy_async();  // Q and the first tile are read by the tensor cores
  tc_fence_before();
  __syncthreads();

  // softmax state of head 16 warp + lane (warps 0..3, lanes 0..15: the rows of an M=64 accumulator)
  const bool head_lane = warp < 4 && lane < 16;
  const int my_h = 16 * (warp & 3) + (lane & 15);
  const float lsc = s_hsc[my_h] * p.logit_scale;
  float m_used = -INFINITY, l_run = 0.f;

  constexpr uint32_t kIdS = idesc_f16(0, 0, 0, 64, kTokU);       // f16, K-major A and B
  constexpr uint32_t kIdSr = idesc_f16(1, 0, 0, 64, kTokU);      // bf16 (RoPE part)
  constexpr uint32_t kIdO = idesc_f16(0, 1, 0, 128, kHeadsU);    // A (latent^T) MN-major
  const uint32_t aQ = smem_addr(sQ), aP = smem_addr(smem + kOffP);
  // S = Q K^T over latent/RoPE buffer `buf`: half 0 takes latent K steps 0..15 into columns kColS,
  // half 1 steps 16..31 and the RoPE part into kColS2 (the softmax adds the two)
  auto issue_s = [&](int buf, int half) {
    const uint32_t aLat = smem_addr(smem + kOffLat + buf * kSizeLat), aRope = smem_addr(smem + kOffRope + buf * kSizeRope);
    const uint32_t d = tmem + (half ? kColS2 : kColS);
#pragma unroll 4
    for (int k = 0; k < kLatU / 32; ++k) {
      const int kk = half * (kLatU / 32) + k;
      umma_f16(d, smem_desc(aQ + kk * 2 * kCore, kCore, (kDqU / 8) * kCore),
               smem_desc(aLat + kk * 2 * kCore, kCore, (kLatU / 8) * kCore), kIdS, k > 0);
    }
    if (half) {
#pragma unroll
      for (int kk = 0; kk < kRopeU / 16; ++kk)
        umma_f16(d, smem_desc(aQ + (kLatU / 8 + 2 * kk) * kCore, kCore, (kDqU / 8) * kCore),
                 smem_desc(aRope + kk * 2 * kCore, kCore, (kRopeU / 8) * kCore), kIdSr, 1u);
    }
    umma_commit(smem_addr(&bar_s));
  };
  // O^T += latent^T P^T over buffer `buf`, M-blocks (latent dims / 128) 2 half .. 2 half + 1
  auto issue_o = [&](int buf, bool first, int half) {
    const uint32_t aLat = smem_addr(smem + kOffLat + buf * kSizeLat);
#pragma unroll
    for (int mt4 = 2 * half; mt4 < 2 * half + 2; ++mt4)
#pragma unroll
      for (int kk = 0; kk < kTokU / 16; ++kk)
        umma_f16(tmem + kColO + mt4 * kHeadsU,
                 smem_desc(aLat + (kk * 2 * (kLatU / 8) + mt4 * 16) * kCore, (kLatU / 8) * kCore, kCore),
                 smem_desc(aP + kk * 2 * kCore, kCore, (kTokU / 8) * kCore), kIdO, (!first || kk > 0) ? 1u : 0u);
    umma_commit(smem_addr(&bar_o));
  };
  const bool s_issuer = lane == 0 && (warp == kWarpS || warp == kWarpS + 1);
  if (s_issuer && n_iter > 0) {
    tc_fence_after();
    issue_s(0, warp - kWarpS);
  }

  for (int it = 0; it < n_iter; ++it) {
    const int buf = it & 1;
    const int count = tile_count(it);
    // PV(it-1) read the other latent buffer and P, and wrote O^T: wait for it before any of them
    // changes; then the next tile goes into the other buffer while S(it) runs on the tensor cores
    if (it > 0) {
      wait_bar(&bar_o, (uint32_t)(it - 1) & 1u);
      tc_fence_after();
    }
    if (it + 1 < n_iter) {
      dequant_tile(regs, smem + kOffLat + (buf ^ 1) * kSizeLat, smem + kOffRope + (buf ^ 1) * kSizeRope, tid);
      if (it + 2 < n_iter) load_tile(regs, base, F, tile_bytes, t_begin + (it + 2) * kTokU, tile_count(it + 2), tid);
    }
    wait_bar(&bar_s, (uint32_t)it & 1u);
    tc_fence_after();

    // ---- softmax rows: lanes 0..15 of warps 0..3 hold head 16 warp + lane
    uint32_t sv0[32], sv1[32];
    if (warp < 4) {
      uint32_t sx[32];
      tmem_ld32(tmem_warp + kColS, sv0);
      tmem_ld32(tmem_warp + kColS + 32, sv1);
      tmem_ld32(tmem_warp + kColS2, sx);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 32; ++t) sv0[t] = __float_as_uint(__uint_as_float(sv0[t]) + __uint_as_float(sx[t]));
      tmem_ld32(tmem_warp + kColS2 + 32, sx);
      tmem_wait_ld();
#pragma unroll
      for (int t = 0; t < 32; ++t) sv1[t] = __float_as_uint(__uint_as_float(sv1[t]) + __uint_as_float(sx[t]));
    }
    int moved = 0;
    if (head_lane) {
      float x[kTokU];
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // four independent chains
#pragma unroll
      for (int t = 0; t < kTokU; ++t) {
        const float sv = __uint_as_float(t < 32 ? sv0[t] : sv1[t - 32]);
        x[t] = t < count ? sv * lsc : -INFINITY;
        m4[t & 3] = fmaxf(m4[t & 3], x[t]);
      }
      const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
      float alpha = 1.f;
      if (mt > m_used + kLazyRescale) {  // also the first tile (m_used = -inf)
        alpha = m_used == -INFINITY ? 0.f : ex2f(m_used - mt);
        m_used = mt;
        l_run *= alpha;
        moved = 1;
      }
      s_alpha[my_h] = alpha;
      float ls4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int tc = 0; tc < kTokU / 8; ++tc) {
        uint32_t h2[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p0 = ex2f(x[8 * tc + 2 * e] - m_used);  // 2^-inf = +0
          const float p1 = ex2f(x[8 * tc + 2 * e + 1] - m_used);
          ls4[e] += p0 + p1;
          const __half2 hp = __floats2half2_rn(p0, p1);
          h2[e] = *reinterpret_cast<const uint32_t*>(&hp);
        }
        *reinterpret_cast<uint4*>(smem + kOffP + core_off(my_h, 8 * tc, kTokU / 8)) = make_uint4(h2[0], h2[1], h2[2], h2[3]);
      }
      l_run += (ls4[0] + ls4[1]) + (ls4[2] + ls4[3]);
    }
    const int any_moved = __syncthreads_or(moved);

    // ---- rescale O^T columns of heads whose maximum moved (not before the first product)
    if (it > 0 && any_moved) {
#pragma unroll 1
      for (int mt4 = 0; mt4 < kLatU / 128; ++mt4) {
        uint32_t r[32];
        const uint32_t ta = tmem_warp + kColO + mt4 * kHeadsU + col_half * 32;
        tmem_ld32(ta, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * s_alpha[col_half * 32 + j]);
        tmem_st32(ta, r);
      }
      tmem_wait_st();
    }
    fence_proxy_async();  // P and the next tile are read by the tensor cores
    tc_fence_before();
    __syncthreads();

    // ---- O^T += latent^T P^T for this tile, then (other threads) S for the next one
    if (warp == kWarpO || warp == kWarpO2) {
      if (lane == 0) {
        tc_fence_after();
        issue_o(buf, it == 0, warp == kWarpO2);
      }
      __syncwarp();
      asm volatile("bar.arrive %0, %1;\n" ::"n"(kIssueBar), "n"(128) : "memory");
    } else if (warp == kWarpS || warp == kWarpS + 1) {
      asm volatile("bar.sync %0, %1;\n" ::"n"(kIssueBar), "n"(128) : "memory");
      if (lane == 0 && it + 1 < n_iter) {
        tc_fence_after();
        issue_s(buf ^ 1, warp - kWarpS);
      }
    }
  }

  // ---- partials (m, l, o) of the 64 heads of this split
  if (n_iter > 0) {
    wait_bar(&bar_o, (uint32_t)(n_iter - 1) & 1u);
    tc_fence_after();
  }
  const int stride = 2 + kLatU;
  float* part = p.part + ((size_t)b * kHeadsU * p.splits + split) * stride;  // head h at + h * splits * stride
  if (head_lane) {
    float* d = part + (size_t)my_h * p.splits * stride;
    d[0] = m_used;
    d[1] = l_run;
  }
#pragma unroll 1
  for (int mt4 = 0; mt4 < kLatU / 128; ++mt4) {
    uint32_t r[32];
    tmem_ld32(tmem_warp + kColO + mt4 * kHeadsU + col_half * 32, r);
    tmem_wait_ld();
    const int dim = 128 * mt4 + 32 * (warp & 3) + lane;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      part[(size_t)(col_half * 32 + j) * p.splits * stride + 2 + dim] = n_iter > 0 ? __uint_as_float(r[j]) : 0.f;
  }

  // ---- teardown: after a wait that gave up, wait once more (bounded) for the last MMAs
  if (tid == 0 && s_fail && n_iter > 0) {
    mbar_wait(smem_addr(&bar_o), (uint32_t)(n_iter - 1) & 1u, p.wait_limit);
    mbar_wait(smem_addr(&bar_s), (uint32_t)(n_iter - 1) & 1u, p.wait_limit);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool mla_umma_supported(const MlaParams& p) {
  return p.fp4.latent == kLatU && p.fp4.rope == kRopeU && p.Hq == kHeadsU && p.chunk % kTokU == 0;
}

cudaError_t launch_decode_mla_umma(const MlaParams& p, cudaStream_t s) {
  const size_t smem = kSmemU;
  cudaError_t e = cudaFuncSetAttribute(decode_mla_umma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_mla_umma<<<dim3(p.splits, p.B), kThreadsU, smem, s>>>(p);
  return launched();
}

}  // namespace kvq
