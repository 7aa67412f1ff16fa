// fp32 SIMT path of the FLARE encode and decode (CUDA cores, FFMA).
//
// Same definitions as the tensor-core path ("FLARE: Fast Low-rank Attention
// Routing Engine" review page, "Основной механизм FLARE": encode
// Z = SDPA(Q, K, V, s=1) with the softmax over tokens, decode
// Y = SDPA(K, Q, Z, s=1) with the softmax over latents), computed in fp32
// throughout so that results stay within 1e-4 of the fp64 definition.
//   encode_f32_kernel: split-token partials in the same (O, mref, l) format as
//                      encode_tc_kernel, merged by lse_merge_kernel.
// Inputs may be stored as bf16 (TQ / TKV / TK = __nv_bfloat16): they are
// widened on load and everything after that is fp32, which is the
// bf16-in / fp32-out mode of the library.
//   decode_f32_kernel: one warp per token; lanes split the latents, the row
//                      max and sum go through warp shuffles, then lanes split
//                      the D output channels.
#pragma once

#include "common.cuh"

namespace flare {

template <typename T>
__device__ __forceinline__ float ld_f32(const T* p);
template <>
__device__ __forceinline__ float ld_f32<float>(const float* p) {
  return *p;
}
template <>
__device__ __forceinline__ float ld_f32<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

struct EncodeF32Args {
  int N, M, q_batched, H, splits, tiles, P;
  const void* Q;  // [H or BH][M][D], TQ
  const void* K;  // [BH][N][D], TKV
  const void* V;
  float* O_part;
  float* m_part;
  float* l_part;
};

constexpr int kF32Tile = 32;  // tokens per smem tile

// grid (splits, BH, row groups); 256 threads; D/min(D,32) threads per latent row.
template <int D, typename TQ, typename TKV>
__global__ void __launch_bounds__(256) encode_f32_kernel(const EncodeF32Args a) {
  constexpr int DPT = D < 32 ? D : 32;  // channels per thread
  constexpr int TPR = D / DPT;          // threads per latent row
  constexpr int RPB = 256 / TPR;        // rows per block
  __shared__ float sK[kF32Tile][D];
  __shared__ float sV[kF32Tile][D];

  const int split = blockIdx.x, bh = blockIdx.y;
  const int row = blockIdx.z * RPB + threadIdx.x / TPR;
  const int part = threadIdx.x % TPR;
  const int d0 = part * DPT;
  const bool active = row < a.M;
  const long long tok0 = static_cast<long long>(split) * a.N / a.splits;
  const long long tok1 = static_cast<long long>(split + 1) * a.N / a.splits;

  float q[DPT], o[DPT];
  const TQ* qrow = static_cast<const TQ*>(a.Q) +
                   ((static_cast<size_t>(a.q_batched ? bh : bh % a.H) * a.M) + (active ? row : 0)) * D;
#pragma unroll
  for (int d = 0; d < DPT; ++d) {
    q[d] = active ? ld_f32(qrow + d0 + d) : 0.f;
    o[d] = 0.f;
  }
  float mref = -INFINITY, l = 0.f;
  const TKV* Kh = static_cast<const TKV*>(a.K) + static_cast<size_t>(bh) * a.N * D;
  const TKV* Vh = static_cast<const TKV*>(a.V) + static_cast<size_t>(bh) * a.N * D;

  for (long long t0 = tok0; t0 < tok1; t0 += kF32Tile) {
    const long long rem = tok1 - t0;
    const int cnt = rem < kF32Tile ? static_cast<int>(rem) : kF32Tile;
    __syncthreads();
    for (int i = threadIdx.x; i < kF32Tile * D; i += blockDim.x) {
      const int j = i / D, d = i % D;
      sK[j][d] = j < cnt ? ld_f32(Kh + (t0 + j) * D + d) : 0.f;
      sV[j][d] = j < cnt ? ld_f32(Vh + (t0 + j) * D + d) : 0.f;
    }
    __syncthreads();
    for (int j = 0; j < cnt; ++j) {
      float dot = 0.f;
#pragma unroll
      for (int d = 0; d < DPT; ++d) dot = fmaf(q[d], sK[j][d0 + d], dot);
#pragma unroll
      for (int w = TPR / 2; w >= 1; w >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, w);
      const float s = dot * kLog2e;
      if (s > mref) {
        const float alpha = exp2f(mref - s);
        l *= alpha;
#pragma unroll
        for (int d = 0; d < DPT; ++d) o[d] *= alpha;
        mref = s;
      }
      const float p = exp2f(s - mref);
      l += p;
#pragma unroll
      for (int d = 0; d < DPT; ++d) o[d] = fmaf(p, sV[j][d0 + d], o[d]);
    }
  }
  if (active) {
    const size_t r = (static_cast<size_t>(bh) * a.P + split) * a.M + row;
#pragma unroll
    for (int d = 0; d < DPT; ++d) a.O_part[r * D + d0 + d] = o[d];
    if (part == 0) {
      a.m_part[r] = mref;
      a.l_part[r] = l;
    }
  }
}

struct DecodeF32Args {
  int N, M, q_batched, H;
  const void* K;   // [BH][N][D], TK
  const float* Q;  // [H or BH][M][D]
  const float* Z;  // [BH][M][D]
  float* Y;        // [BH][N][D]
};

// grid (ceil(N / 8), BH); 256 threads = 8 warps, one token per warp.
template <int D, typename TK>
__global__ void __launch_bounds__(256) decode_f32_kernel(const DecodeF32Args a) {
  __shared__ float sk[8][D];
  __shared__ float sp[8][256];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const long long tok = static_cast<long long>(blockIdx.x) * 8 + warp;
  if (tok >= a.N) return;  // whole warp leaves together
  const TK* k = static_cast<const TK*>(a.K) + (static_cast<size_t>(bh) * a.N + tok) * D;
  for (int d = lane; d < D; d += 32) sk[warp][d] = ld_f32(k + d);
  __syncwarp();
  const float* Q = a.Q + static_cast<size_t>(a.q_batched ? bh : bh % a.H) * a.M * D;
  const float* Z = a.Z + static_cast<size_t>(bh) * a.M * D;

  float s[8];  // latents lane, lane+32, ... (M <= 256)
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int m = lane + 32 * j;
    s[j] = -INFINITY;
    if (m < a.M) {
      float dot = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) dot = fmaf(sk[warp][d], __ldg(Q + m * D + d), dot);
      s[j] = dot * kLog2e;
      mx = fmaxf(mx, s[j]);
    }
  }
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, w));
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int m = lane + 32 * j;
    if (m < a.M) {
      const float p = exp2f(s[j] - mx);
      sum += p;
      sp[warp][m] = p;
    }
  }
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, w);
  __syncwarp();
  const float inv = 1.f / sum;
  float* y = a.Y + (static_cast<size_t>(bh) * a.N + tok) * D;
  for (int d = lane; d < D; d += 32) {
    float acc = 0.f;
    for (int m = 0; m < a.M; ++m) acc = fmaf(sp[warp][m], __ldg(Z + m * D + d), acc);
    y[d] = acc * inv;
  }
}

}  // namespace flare
