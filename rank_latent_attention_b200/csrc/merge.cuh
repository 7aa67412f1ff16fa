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
// exchanged).  Partials with l_p = 0 (no tokens) are skipped.  The same kernel
// combines the per-device (O, lse) results of a token-sharded encode.
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

// Where the partials of (bh, p) sit, in floats: O element (m, d) at
// O_part[bh * o_head + p * o_part + m * D + d], its statistics at
// [bh * s_head + p * s_part + m].  The encode's own workspace is [BH][P][M][D]
// (o_head = P*M*D, o_part = M*D, s_head = P*M, s_part = M); the per-device
// results of a token-sharded encode, gathered, are [R][BH][M][D] with any
// stride between devices (o_head = M*D, s_head = M, o_part = s_part = the
// stride).
struct MergeGeom {
  int P, M, D;
  long long o_head, o_part, s_head, s_part;
};

// grid (ceil(M*D / 256), BH), 256 threads; one thread per output element.
//
// FROM_LSE = false: partials are (O_p unnormalised, mref_p log2-domain, l_p).
// FROM_LSE = true:  partials are (O_p normalised, lse_p natural log) -- one
//   token shard's softmax output and log-sum-exp; an empty shard has
//   lse_p = -inf.  l_part is unused; mref_p = lse_p log2(e), l_p = 1.
// lse_out (may be null) receives the natural-log log-sum-exp of the union,
// ln(2^m* sum_p w_p l_p); a row with no tokens at all gets out = 0 and
// lse_out = -inf.
// split (may be null; fp32 out only): {hi, lo} receive the result as a bf16
// pair, hi = bf16(out), lo = bf16(out - hi), the operand form of the next
// step's split-precision MMAs.
struct SplitOut {
  __nv_bfloat16* hi;
  __nv_bfloat16* lo;
};
template <typename OutT, bool FROM_LSE>
__global__ void __launch_bounds__(256) lse_merge_kernel(const float* __restrict__ O_part,
                                                        const float* __restrict__ m_part,
                                                        const float* __restrict__ l_part, OutT* __restrict__ out,
                                                        float* __restrict__ lse_out, MergeGeom g,
                                                        SplitOut split = SplitOut{nullptr, nullptr}) {
  constexpr float kLn2 = 0.6931471805599453f;
  // launched with programmatic serialisation after the encode that writes
  // the partials: let the next kernel start its prologue, wait for the
  // partials
  ptx::grid_dep_launch();
  ptx::grid_dep_wait();
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= g.M * g.D) return;
  const int bh = blockIdx.y;
  const int m = idx / g.D;
  const int d = idx - m * g.D;
  const long long sbase = bh * g.s_head + m;
  const long long obase = bh * g.o_head + static_cast<long long>(m) * g.D + d;
  // One pass with a running maximum: a partial whose reference lies above
  // the running one rescales the sums so far (exact; usually only the first
  // few partials do).  The loads of a batch of partials are independent, so
  // they are issued together instead of one dependent round trip each.
  float mx = -INFINITY, num = 0.f, den = 0.f;
  constexpr int kBatch = 8;
  for (int p0 = 0; p0 < g.P; p0 += kBatch) {
    float mp[kBatch], lp[kBatch], op[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int p = p0 + u;
      mp[u] = -INFINITY;
      lp[u] = 0.f;
      op[u] = 0.f;
      if (p < g.P) {
        const long long row = sbase + p * g.s_part;
        if constexpr (FROM_LSE) {
          const float lse = m_part[row];
          mp[u] = lse * kLog2e;
          lp[u] = lse > -INFINITY ? 1.f : 0.f;
        } else {
          mp[u] = m_part[row];
          lp[u] = l_part[row];
        }
        op[u] = O_part[obase + p * g.o_part];
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (lp[u] > 0.f) {  // partials without tokens carry no weight
        if (mp[u] > mx) {
          const float scale = mx > -INFINITY ? exp2f(mx - mp[u]) : 0.f;
          num *= scale;
          den *= scale;
          mx = mp[u];
        }
        const float w = exp2f(mp[u] - mx);
        den = fmaf(w, lp[u], den);
        num = fmaf(w, op[u], num);
      }
    }
  }
  const size_t orow = static_cast<size_t>(bh) * g.M + m;
  const float v = den > 0.f ? num / den : 0.f;
  out[orow * g.D + d] = to_out<OutT>(v);
  if (split.hi) {
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    split.hi[orow * g.D + d] = h;
    split.lo[orow * g.D + d] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
  if (lse_out && d == 0) lse_out[orow] = den > 0.f ? (mx + log2f(den)) * kLn2 : -INFINITY;
}

}  // namespace flare
