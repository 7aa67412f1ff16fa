// Log-sum-exp merge of split-token encode partials.
//
// For each (b, h) and latent m, with P partials (O_p, mref_p, l_p) that each
// cover a disjoint range of tokens (log2-domain reference maxima):
//   m* = max_p mref_p,  w_p = 2^(mref_p - m*),
//   out[m][:] = sum_p w_p O_p[m][:] / sum_p w_p l_p.
// This is the exact combination of per-shard softmax statistics that the
// FLARE++ page describes for its token-sharded encoder ("FLARE++: Low-rank
// attention with dynamic attention routing", "Contributions Clés",
// context-parallel item: only latent outputs and softmax statistics are
// exchanged).  Partials with l_p = 0 (no tokens) are skipped.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace flare {

template <typename OutT>
__device__ __forceinline__ OutT to_out(float v);
template <>
__device__ __forceinline__ float to_out<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// grid (ceil(M*D / 256), BH), 256 threads; one thread per output element.
template <typename OutT>
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* __restrict__ O_part,
                                                        const float* __restrict__ m_part,
                                                        const float* __restrict__ l_part, OutT* __restrict__ out,
                                                        int P, int M, int D) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= M * D) return;
  const int bh = blockIdx.y;
  const int m = idx / D;
  const int d = idx - m * D;
  const size_t base = static_cast<size_t>(bh) * P;
  float mx = -INFINITY;
  for (int p = 0; p < P; ++p) {
    const size_t row = (base + p) * M + m;
    if (l_part[row] > 0.f) mx = fmaxf(mx, m_part[row]);
  }
  float num = 0.f, den = 0.f;
  for (int p = 0; p < P; ++p) {
    const size_t row = (base + p) * M + m;
    const float l = l_part[row];
    if (l > 0.f) {
      const float w = exp2f(m_part[row] - mx);
      den = fmaf(w, l, den);
      num = fmaf(w, O_part[row * D + d], num);
    }
  }
  out[(static_cast<size_t>(bh) * M + m) * D + d] = to_out<OutT>(num / den);
}

}  // namespace flare
