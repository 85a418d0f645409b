// Merge of softmax states computed over disjoint parts of the context (context-parallel decode:
// each rank, or each cache shard, attends over its own tokens). For a query head, part i holds
// m_i (its largest logit, log2 units), l_i = sum 2^(l_t - m_i) and o_i = sum 2^(l_t - m_i) v_t over
// its tokens; softmax over the union of the parts is
//   out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i,   M = max_i m_i,
// the same log-sum-exp combine the split reduce applies to a single cache's splits. A part with no
// tokens has m = -inf, l = 0, o = 0 and drops out; all parts empty gives an all-zero output.
#include "kvq_internal.h"

namespace kvq {
namespace {

__global__ void combine_partials(const float* __restrict__ parts, int n_parts, int rows, int dv,
                                 float* __restrict__ out) {
  const int row = blockIdx.x;
  const size_t stride = 2 + (size_t)dv, part_stride = (size_t)rows * stride;
  const float* base = parts + (size_t)row * stride;
  float M = -INFINITY;
  for (int i = 0; i < n_parts; ++i) M = fmaxf(M, base[i * part_stride]);
  for (int c = threadIdx.x; c < dv; c += blockDim.x) {
    float L = 0.f, o = 0.f;
    for (int i = 0; i < n_parts; ++i) {
      const float* pi = base + i * part_stride;
      const float w = pi[0] == -INFINITY ? 0.f : exp2f(pi[0] - M);
      L = fmaf(w, pi[1], L);
      o = fmaf(w, pi[2 + c], o);
    }
    out[(size_t)row * dv + c] = L > 0.f ? o / L : 0.f;
  }
}

}  // namespace

cudaError_t launch_combine_partials(const float* parts, int n_parts, int rows, int dv, float* out, cudaStream_t s) {
  combine_partials<<<rows, dv < 512 ? 128 : 256, 0, s>>>(parts, n_parts, rows, dv, out);
  return launched();
}

}  // namespace kvq
