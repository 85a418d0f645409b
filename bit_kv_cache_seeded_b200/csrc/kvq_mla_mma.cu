// Tensor-core split-K decode attention over an FP4 MLA-style latent cache.
//
// "How DeepSeek-V4.1-Flash cut KV cache storage by 4x via CSA2": one 512-dim latent per token
// is shared by all heads (section "CSA2") and stored as FP4 E2M1 with one scale per 16
// channels (section "Numerics and hardware efficiency"; the scale is an E4M3 byte here). With
// the absorbed query q = [q_lat ; q_rope], 64 heads share every token, so decode attention is
// a pair of dense contractions per 64-token tile:
//   S = Q [64 heads x 576] . K^T,   K_t = [latent_hat_t (512) ; k_rope_t (64)]
//   O += P [64 heads x 64 tokens] . latent_hat [64 tokens x 512]
// latent_hat = E4M3 scale x E2M1 value has at most 6 significant bits and lies in
// [2^-10, 2688], so it is exact in f16: the tile is dequantised with cvt.rn.f16x2.e2m1x2 and a
// packed f16 multiply by the scale (cvt.rn.f16x2.e4m3x2). Q's latent part is scaled per head by
// a power of two (exact) into f16 range; the RoPE part stays bf16 and uses bf16 MMAs into the
// same accumulators. P is rounded to f16 (2^-11 relative), accumulation is fp32 throughout.
//
// CTA: 8 warps, 64 tokens per iteration, cp.async double buffering of the packed tiles.
// Warp w owns heads 16 (w % 4) .. +15: in QK it takes tokens 32 (w / 4) .. +31, in PV it takes
// channels 256 (w / 4) .. +255. Partials (m, l, o[512]) per (sequence, head, split) go to the
// workspace in the format of the CUDA-core kernel; the same reduce kernel finishes.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kWarpsL = 8;
constexpr int kThreadsL = kWarpsL * 32;
constexpr int kTokL = 64;          // tokens per CTA iteration (two cache tiles)
constexpr int kLat = 512, kRope = 64, kDq = kLat + kRope;
constexpr int kHeadsL = 64;
// padded smem row strides (bytes): +16 B per row keeps 8 consecutive rows on distinct banks
constexpr int kQStride = kDq * 2 + 16;       // Q rows: 512 f16 + 64 bf16
constexpr int kLatStride = kLat * 2 + 16;    // dequantised latent rows (f16)
constexpr int kRopeStride = kRope * 2 + 16;  // RoPE key rows (bf16)
constexpr int kPStride = kTokL * 2 + 16;     // P rows (f16)

__device__ __forceinline__ unsigned smem_u32(const void* p) { return (unsigned)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void ldsm_x4(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(unsigned addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
               : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
               : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
// Two E2M1 codes (one byte, channel 2k in the low nibble) to f16x2 (channel 2k in the low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{\n .reg .b8 b;\n cvt.u8.u32 b, %1;\n cvt.rn.f16x2.e2m1x2 %0, b;\n}\n" : "=r"(r) : "r"(byte));
  return r;
}
// Two E4M3 bytes (low 16 bits) to f16x2.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(r) : "h"((unsigned short)two));
  return r;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
__device__ __forceinline__ void cp_async16l(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem));
}
__device__ __forceinline__ float exp2_diffl(float a, float b) { return (a == -INFINITY) ? 0.f : exp2f(a - b); }

__global__ void __launch_bounds__(kThreadsL, 1)
decode_mla_mma(const __grid_constant__ MlaParams p) {
  extern __shared__ __align__(16) unsigned char smem[];
  const Fp4Layout& F = p.fp4;
  const int tile_bytes = F.tile_bytes;
  unsigned char* qs = smem;                                   // [64][kQStride]
  unsigned char* lat = qs + kHeadsL * kQStride;               // [64 tokens][kLatStride]
  unsigned char* rope = lat + kTokL * kLatStride;             // [64 tokens][kRopeStride]
  unsigned char* ps = rope + kTokL * kRopeStride;             // [64 heads][kPStride]
  unsigned char* raw = ps + kHeadsL * kPStride;               // [2 stages][2 cache tiles]
  float* red = reinterpret_cast<float*>(raw + 2 * 2 * tile_bytes);  // [8 warps][16]
  float* hsc = red + kWarpsL * 16;                            // [64] per-head query scale

  const int split = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int mt = warp & 3, half = warp >> 2;  // head block, token half (QK) / channel half (PV)
  const int len = p.lens[b];
  const int t_begin = split * p.chunk;
  const int t_end = min(len, t_begin + p.chunk);
  const int n_iter = t_end > t_begin ? (t_end - t_begin + kTokL - 1) / kTokL : 0;
  const unsigned char* base = reinterpret_cast<const unsigned char*>(p.reg) + (size_t)b * p.tiles_per_seq * tile_bytes;

  auto load_stage = [&](int it) {
    if (it < n_iter) {
      const int tile0 = (t_begin + it * kTokL) / kTile;
      const int ntiles = (t_begin + it * kTokL + kTile < t_end) ? 2 : 1;
      unsigned char* dst = raw + (it & 1) * 2 * tile_bytes;
      const unsigned char* src = base + (size_t)tile0 * tile_bytes;
      for (int c = tid; c < ntiles * tile_bytes / 16; c += kThreadsL) cp_async16l(dst + 16 * c, src + 16 * c);
    }
    asm volatile("cp.async.commit_group;\n" ::);
  };
  load_stage(0);

  // ---- query: per-head power-of-two scale into f16 range; latent part f16, RoPE part bf16
  const int Hq = p.Hq;
  const size_t qbase = (size_t)b * Hq * kDq;
  for (int h = warp; h < kHeadsL; h += kWarpsL) {
    float mx = 0.f;
    if (h < Hq)
      for (int c = lane; c < kDq; c += 32) {
        const float v = p.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[qbase + (size_t)h * kDq + c])
                               : reinterpret_cast<const float*>(p.q)[qbase + (size_t)h * kDq + c];
        mx = fmaxf(mx, fabsf(v));
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float sc = mx > 0.f ? exp2f(ceilf(log2f(mx)) - 14.f) : 1.f;
    if (lane == 0) hsc[h] = sc;
    const float inv = 1.f / sc;
    for (int c = lane; c < kDq; c += 32) {
      float v = 0.f;
      if (h < Hq)
        v = p.bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q)[qbase + (size_t)h * kDq + c])
                   : reinterpret_cast<const float*>(p.q)[qbase + (size_t)h * kDq + c];
      v *= inv;
      if (c < kLat) reinterpret_cast<__half*>(qs + h * kQStride)[c] = __float2half_rn(v);
      else reinterpret_cast<__nv_bfloat16*>(qs + h * kQStride)[c] = __float2bfloat16_rn(v);
    }
  }
  __syncthreads();

  // per-thread constants: heads of rows g and g+8 of this warp's head block
  const int h0 = 16 * mt + g, h1 = h0 + 8;
  const float lsc0 = hsc[h0] * p.logit_scale, lsc1 = hsc[h1] * p.logit_scale;
  float m_run0 = -INFINITY, m_run1 = -INFINITY, l_run0 = 0.f, l_run1 = 0.f;
  float o[32][4];
#pragma unroll
  for (int nt = 0; nt < 32; ++nt)
#pragma unroll
    for (int c = 0; c < 4; ++c) o[nt][c] = 0.f;

  // ldmatrix row addresses (per thread) for A fragments (row-major [row][k])
  const int a_row = (lane & 7) + 8 * ((lane >> 3) & 1), a_col = 8 * (lane >> 4);
  const unsigned q_addr = smem_u32(qs + (16 * mt + a_row) * kQStride + a_col * 2);
  const unsigned p_addr = smem_u32(ps + (16 * mt + a_row) * kPStride + a_col * 2);
  // B fragments from [token][k] rows (QK): rows n = (lane & 7) + 8 * (lane >> 4), k = 8 * ((lane >> 3) & 1)
  const int b_row = (lane & 7) + 8 * (lane >> 4), b_col = 8 * ((lane >> 3) & 1);
  // B fragments from [token][channel] rows (PV, transposed): token = a_row, channel = a_col

  for (int it = 0; it < n_iter; ++it) {
    load_stage(it + 1);
    asm volatile("cp.async.wait_group 1;\n" ::);
    __syncthreads();
    const unsigned char* rt = raw + (it & 1) * 2 * tile_bytes;
    const int count = min(kTokL, t_end - (t_begin + it * kTokL));

    // ---- dequantise the tile: thread -> (token, 32 channels); RoPE copied
    {
      const int tok = tid >> 2, part = tid & 3;  // 64 tokens x 4 parts of 128 channels
      const unsigned char* ct = rt + (tok / kTile) * tile_bytes;
      const int slot = tok % kTile;
      uint4* dst = reinterpret_cast<uint4*>(lat + tok * kLatStride + part * 256);
      if (tok < count) {
        const uint4* codes = reinterpret_cast<const uint4*>(ct + F.off_codes + slot * (kLat / 2) + part * 64);
        const uint2 scl = *reinterpret_cast<const uint2*>(ct + F.off_scales + slot * (kLat / 16) + part * 8);
        // scales of groups (2q, 2q+1) as f16x2, q = 0..3 (8 groups of 16 channels in this part)
        const uint32_t spair[4] = {e4m3x2_to_f16x2(scl.x & 0xFFFFu), e4m3x2_to_f16x2(scl.x >> 16),
                                   e4m3x2_to_f16x2(scl.y & 0xFFFFu), e4m3x2_to_f16x2(scl.y >> 16)};
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {  // 16 bytes = 32 channels = groups 2 q4 and 2 q4 + 1
          const uint4 c = codes[q4];
          const uint32_t w[4] = {c.x, c.y, c.z, c.w};
          const uint32_t slo = spair[q4] & 0xFFFFu, shi = spair[q4] >> 16;
          const uint32_t bA = slo | (slo << 16), bB = shi | (shi << 16);  // broadcast f16 scales
          uint32_t out[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint32_t byte = (w[k >> 2] >> (8 * (k & 3))) & 0xFFu;
            out[k] = hmul2(e2m1x2_to_f16x2(byte), k < 8 ? bA : bB);
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[4 * q4 + v] = make_uint4(out[4 * v], out[4 * v + 1], out[4 * v + 2], out[4 * v + 3]);
        }
      } else {
#pragma unroll
        for (int v = 0; v < 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
      }
      if (part == 0) {
        const uint4* rs = reinterpret_cast<const uint4*>(ct + F.off_rope + slot * (kRope * 2));
        uint4* rd = reinterpret_cast<uint4*>(rope + tok * kRopeStride);
#pragma unroll
        for (int v = 0; v < 8; ++v) rd[v] = tok < count ? rs[v] : make_uint4(0, 0, 0, 0);
      }
    }
    __syncthreads();

    // ---- S = Q K^T for heads 16 mt.., tokens 32 half..
    float s[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[nt][c] = 0.f;
    {
      const unsigned k_addr0 = smem_u32(lat + (32 * half + b_row) * kLatStride + b_col * 2);
      const unsigned k_addr1 = k_addr0 + 16 * kLatStride;
#pragma unroll 4
      for (int ks = 0; ks < kLat / 16; ++ks) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3, b4, b5, b6, b7;
        ldsm_x4(q_addr + ks * 32, a0, a1, a2, a3);
        ldsm_x4(k_addr0 + ks * 32, b0, b1, b2, b3);
        ldsm_x4(k_addr1 + ks * 32, b4, b5, b6, b7);
        mma_f16(s[0], a0, a1, a2, a3, b0, b1);
        mma_f16(s[1], a0, a1, a2, a3, b2, b3);
        mma_f16(s[2], a0, a1, a2, a3, b4, b5);
        mma_f16(s[3], a0, a1, a2, a3, b6, b7);
      }
      const unsigned r_addr0 = smem_u32(rope + (32 * half + b_row) * kRopeStride + b_col * 2);
      const unsigned r_addr1 = r_addr0 + 16 * kRopeStride;
#pragma unroll
      for (int ks = 0; ks < kRope / 16; ++ks) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3, b4, b5, b6, b7;
        ldsm_x4(q_addr + kLat * 2 + ks * 32, a0, a1, a2, a3);
        ldsm_x4(r_addr0 + ks * 32, b0, b1, b2, b3);
        ldsm_x4(r_addr1 + ks * 32, b4, b5, b6, b7);
        mma_bf16(s[0], a0, a1, a2, a3, b0, b1);
        mma_bf16(s[1], a0, a1, a2, a3, b2, b3);
        mma_bf16(s[2], a0, a1, a2, a3, b4, b5);
        mma_bf16(s[3], a0, a1, a2, a3, b6, b7);
      }
    }
    // logits (base 2), masked; per-warp row maxima over its 32 tokens
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const int tk = 32 * half + 8 * nt + 2 * t;
      s[nt][0] = tk < count ? s[nt][0] * lsc0 : -INFINITY;
      s[nt][1] = tk + 1 < count ? s[nt][1] * lsc0 : -INFINITY;
      s[nt][2] = tk < count ? s[nt][2] * lsc1 : -INFINITY;
      s[nt][3] = tk + 1 < count ? s[nt][3] * lsc1 : -INFINITY;
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
#pragma unroll
    for (int o2 = 1; o2 < 4; o2 <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o2));
    }
    if (t == 0) { red[warp * 16 + g] = mx0; red[warp * 16 + g + 8] = mx1; }
    __syncthreads();
    const int other = warp ^ 4;
    const float mn0 = fmaxf(m_run0, fmaxf(mx0, red[other * 16 + g]));
    const float mn1 = fmaxf(m_run1, fmaxf(mx1, red[other * 16 + g + 8]));
    const float c0 = exp2_diffl(m_run0, mn0), c1 = exp2_diffl(m_run1, mn1);
    m_run0 = mn0;
    m_run1 = mn1;
    float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 4; ++nt) {
      const float p0 = exp2_diffl(s[nt][0], mn0), p1 = exp2_diffl(s[nt][1], mn0);
      const float p2 = exp2_diffl(s[nt][2], mn1), p3 = exp2_diffl(s[nt][3], mn1);
      ls0 += p0 + p1;
      ls1 += p2 + p3;
      const int tk = 32 * half + 8 * nt + 2 * t;
      *reinterpret_cast<__half2*>(ps + h0 * kPStride + tk * 2) = __floats2half2_rn(p0, p1);
      *reinterpret_cast<__half2*>(ps + h1 * kPStride + tk * 2) = __floats2half2_rn(p2, p3);
    }
    l_run0 = l_run0 * c0 + ls0;  // partial over this warp's token half; halves summed at the end
    l_run1 = l_run1 * c1 + ls1;
#pragma unroll
    for (int nt = 0; nt < 32; ++nt) {
      o[nt][0] *= c0; o[nt][1] *= c0;
      o[nt][2] *= c1; o[nt][3] *= c1;
    }
    __syncthreads();

    // ---- O += P V for heads 16 mt.., channels 256 half..
#pragma unroll
    for (int ks = 0; ks < kTokL / 16; ++ks) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(p_addr + ks * 32, a0, a1, a2, a3);
      const unsigned v_addr = smem_u32(lat + (16 * ks + a_row) * kLatStride + (256 * half + a_col) * 2);
#pragma unroll
      for (int np = 0; np < 16; ++np) {  // pairs of n8 tiles (16 channels)
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(v_addr + np * 32, b0, b1, b2, b3);
        mma_f16(o[2 * np], a0, a1, a2, a3, b0, b1);
        mma_f16(o[2 * np + 1], a0, a1, a2, a3, b2, b3);
      }
    }
  }

  // ---- partials
  asm volatile("cp.async.wait_group 0;\n" ::);
#pragma unroll
  for (int o2 = 1; o2 < 4; o2 <<= 1) {
    l_run0 += __shfl_xor_sync(0xffffffffu, l_run0, o2);
    l_run1 += __shfl_xor_sync(0xffffffffu, l_run1, o2);
  }
  __syncthreads();
  if (t == 0) { red[warp * 16 + g] = l_run0; red[warp * 16 + g + 8] = l_run1; }
  __syncthreads();
  const int stride = 2 + kLat;
  if (h0 < Hq) {
    float* d0 = p.part + (((size_t)b * Hq + h0) * p.splits + split) * stride;
    float* d1 = p.part + (((size_t)b * Hq + h1) * p.splits + split) * stride;
    if (half == 0 && t == 0) {
      d0[0] = m_run0; d0[1] = red[warp * 16 + g] + red[(warp ^ 4) * 16 + g];
      d1[0] = m_run1; d1[1] = red[warp * 16 + g + 8] + red[(warp ^ 4) * 16 + g + 8];
    }
#pragma unroll
    for (int nt = 0; nt < 32; ++nt) {
      const int ch = 256 * half + 8 * nt + 2 * t;
      *reinterpret_cast<float2*>(d0 + 2 + ch) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(d1 + 2 + ch) = make_float2(o[nt][2], o[nt][3]);
    }
  }
}

}  // namespace

size_t mla_mma_smem_bytes(int tile_bytes) {
  size_t s = (size_t)kHeadsL * kQStride + (size_t)kTokL * kLatStride + (size_t)kTokL * kRopeStride +
             (size_t)kHeadsL * kPStride + (size_t)2 * 2 * tile_bytes + sizeof(float) * (kWarpsL * 16 + kHeadsL);
  return (s + 15) / 16 * 16;
}

bool mla_mma_supported(const MlaParams& p) {
  return p.fp4.latent == kLat && p.fp4.rope == kRope && p.Hq % 16 == 0 && p.Hq <= kHeadsL && p.chunk % kTokL == 0;
}

cudaError_t launch_decode_mla_mma(const MlaParams& p, cudaStream_t s) {
  const size_t smem = mla_mma_smem_bytes(p.fp4.tile_bytes);
  cudaError_t e = cudaFuncSetAttribute(decode_mla_mma, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  decode_mla_mma<<<dim3(p.splits, p.B), kThreadsL, smem, s>>>(p);
  return launched();
}

}  // namespace kvq
