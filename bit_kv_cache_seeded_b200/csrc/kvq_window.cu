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
// window_part (kvq_window.cuh) over the sink and recent tokens, in the split kernel's extra CTAs or
// in window_decode below; the reduce merges the window's softmax states (m, l, o_r) with the splits'.
#include <cuda_bf16.h>

#include "kvq_internal.h"
#include "kvq_window.cuh"

namespace kvq {
namespace {

constexpr int kWinThreads = 256;

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

// One CTA of four warps per (window part, kv-head, sequence): the whole query group.
template <int GH>
__global__ void __launch_bounds__(128) window_decode(const __grid_constant__ DecodeParams p) {
  __shared__ __align__(16) float sm[window_smem_floats<4, GH>()];
  window_part<4, GH>(p, blockIdx.z, blockIdx.y, 0, blockIdx.x, sm);
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
  const dim3 grid(p.win_parts, p.Hkv, p.B);
  switch (p.group) {
    case 1: window_decode<1><<<grid, 128, 0, s>>>(p); break;
    case 2: window_decode<2><<<grid, 128, 0, s>>>(p); break;
    case 4: window_decode<4><<<grid, 128, 0, s>>>(p); break;
    case 8: window_decode<8><<<grid, 128, 0, s>>>(p); break;
    default: return cudaErrorNotSupported;
  }
  return launched();
}

}  // namespace kvq
