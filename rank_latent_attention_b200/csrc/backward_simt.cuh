// Backward of the FLARE++ mixer on the CUDA cores (fp32 arithmetic).
//
// Forward per head (b, h), scale 1 ("FLARE++: Low-rank attention with dynamic
// attention routing", "Méthodologie : FLARE++"; the encode and decode forms of
// the "FLARE" review page, "Основной механизм FLARE"):
//   S1 = Q~ K^T,  A1 = softmax over tokens,  Q_dyn = A1 V
//   S2 = Q_dyn K^T, A2 = softmax over tokens, Z = A2 V
//   S3 = K Q_dyn^T, P3 = softmax over latents, Y = P3 Z
// Gradients of L = sum(dY * Y), last step first:
//   dZ = P3^T dY;  dS3 = P3 (dY Z^T - delta),  delta_n = dY_n . Y_n
//   dS2 = A2 (dZ V^T - c2),  c2_m = dZ_m . Z_m
//   dQ_dyn = dS3^T K + dS2 K
//   dS1 = A1 (dQ_dyn V^T - c1),  c1_m = dQ_dyn_m . Q_dyn_m
//   d_seeds = sum_b dS1 K
//   dK = (dS3 + dS2^T) Q_dyn + dS1^T Q~        (S3 = S2^T: one logit serves both)
//   dV = A2^T dZ + A1^T dQ_dyn
//
// Every softmax is rebuilt from its log-sum-exp: lse1, lse2 per latent (from
// the recomputed encodes) and lse3 per token (token_stats_kernel).  With those
// and the row terms delta, c1, c2 known, each pass splits freely over latent
// and token chunks:
//   token_stats_kernel     lse3_n, delta_n                     (token rows)
//   latent_grad_kernel     DEC:  dZ, dQ_dyn(decode) partials   (latent rows)
//                          ENC:  dQ_dyn(routing) / d_seeds partials
//   grad_reduce_kernel     sums the partials, forms c2 / c1
//   token_grad_kernel      dK, dV                              (token rows)
// Inputs T (seeds, K, V, dY, Q_dyn, Z) are fp32 or bf16 storage; everything
// is computed and accumulated in fp32 and only dK, dV and d_seeds are stored
// back in T.
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"
#include "simt_f32.cuh"

namespace flare {

constexpr int kBwdChunk = 32;  // latents per chunk = tokens per tile
constexpr int kBwdThreads = 256;

template <typename T>
__device__ __forceinline__ void st_from_f32(T* p, float v);
template <>
__device__ __forceinline__ void st_from_f32<float>(float* p, float v) {
  *p = v;
}
template <>
__device__ __forceinline__ void st_from_f32<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

// rows [r0, r0 + 32) of a [rows][D] matrix into smem [32][D + 1] as fp32;
// rows past `rows` read as 0.
template <int D, typename T>
__device__ __forceinline__ void load_rows(float* dst, const T* src, long long r0, long long rows) {
  for (int i = threadIdx.x; i < kBwdChunk * D; i += blockDim.x) {
    const int r = i / D, d = i - (i / D) * D;
    dst[r * (D + 1) + d] = (r0 + r < rows) ? ld_f32(src + (r0 + r) * D + d) : 0.f;
  }
}

template <int D>
__device__ __forceinline__ float dot_rows(const float* a, const float* b) {
  float acc = 0.f;
#pragma unroll 16
  for (int d = 0; d < D; ++d) acc = fmaf(a[d], b[d], acc);
  return acc;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, w));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) v += __shfl_xor_sync(0xffffffffu, v, w);
  return v;
}

struct BwdArgs {
  int N, M, H;
  const void* seeds;  // [H][M][D]
  const void* K;      // [BH][N][D]
  const void* V;
  const void* dY;
  const void* Qd;     // [BH][M][D]  Q_dyn as the forward stored it
  const void* Z;      // [BH][M][D]
  const float* lse1;  // [BH][M]
  const float* lse2;  // [BH][M]
  float* lse3;        // [BH][N]
  float* delta;       // [BH][N]
  float* dZ;          // [BH][M][D]
  float* dQd;         // [BH][M][D]
  float* c1;          // [BH][M]
  float* c2;          // [BH][M]
  __nv_bfloat16* dZ16;   // [BH][M][D] bf16 copies of dZ and dQ_dyn for tensor-core
  __nv_bfloat16* dQd16;  // operands (null when the CUDA-core token kernel runs)
  float* part;        // [BH][S][M][D] x 2 (second block at part + part_stride)
  float* exch;        // token-sharded backward: the sums each rank contributes, summed over ranks
                      // between phases ([BH][M][D] x 2 after the decode pass, then x 1, then [H][M][D])
  long long part_stride;
  int S;              // token splits of the latent-row kernels
  void* d_seeds;      // [H][M][D]
  void* dK;           // [BH][N][D]
  void* dV;
};

// ---------------------------------------------------------------- token stats
// grid (ceil(N / 32), BH); 256 threads.  Warp w takes tokens w, w + 8, ...
// of the tile; lanes take the latents of a chunk.  Online over the chunks:
// running max, sum of exps and sum of exp * (dY_n . Z_m) per token.
template <int D, typename T>
__global__ void __launch_bounds__(kBwdThreads) token_stats_kernel(const BwdArgs a) {
  extern __shared__ float sm[];
  float* sK = sm;                            // [32][D+1]
  float* sG = sK + kBwdChunk * (D + 1);      // dY tile
  float* sQ = sG + kBwdChunk * (D + 1);      // Q_dyn chunk
  float* sZ = sQ + kBwdChunk * (D + 1);      // Z chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const long long t0 = static_cast<long long>(blockIdx.x) * kBwdChunk;
  const size_t tok_base = static_cast<size_t>(bh) * a.N;
  load_rows<D>(sK, static_cast<const T*>(a.K) + tok_base * D, t0, a.N);
  load_rows<D>(sG, static_cast<const T*>(a.dY) + tok_base * D, t0, a.N);
  const T* Qh = static_cast<const T*>(a.Qd) + static_cast<size_t>(bh) * a.M * D;
  const T* Zh = static_cast<const T*>(a.Z) + static_cast<size_t>(bh) * a.M * D;

  constexpr int kPerWarp = kBwdChunk / 8;
  float mx[kPerWarp], l[kPerWarp], acc[kPerWarp];
#pragma unroll
  for (int j = 0; j < kPerWarp; ++j) {
    mx[j] = -INFINITY;
    l[j] = 0.f;
    acc[j] = 0.f;
  }
  for (int m0 = 0; m0 < a.M; m0 += kBwdChunk) {
    __syncthreads();
    load_rows<D>(sQ, Qh, m0, a.M);
    load_rows<D>(sZ, Zh, m0, a.M);
    __syncthreads();
    const bool live = m0 + lane < a.M;
#pragma unroll
    for (int j = 0; j < kPerWarp; ++j) {
      const int t = warp + 8 * j;
      const float s = live ? dot_rows<D>(sK + t * (D + 1), sQ + lane * (D + 1)) : -INFINITY;
      const float g = live ? dot_rows<D>(sG + t * (D + 1), sZ + lane * (D + 1)) : 0.f;
      const float cm = warp_max(s);
      const float nm = fmaxf(mx[j], cm);
      const float scale = mx[j] == -INFINITY ? 0.f : expf(mx[j] - nm);
      const float e = live ? expf(s - nm) : 0.f;
      l[j] = l[j] * scale + warp_sum(e);
      acc[j] = acc[j] * scale + warp_sum(e * g);
      mx[j] = nm;
    }
  }
  if (lane == 0) {
#pragma unroll
    for (int j = 0; j < kPerWarp; ++j) {
      const long long t = t0 + warp + 8 * j;
      if (t < a.N) {
        a.lse3[tok_base + t] = mx[j] + logf(l[j]);
        a.delta[tok_base + t] = acc[j] / l[j];
      }
    }
  }
}

// ---------------------------------------------------------------- latent rows
// grid (S, BH, ceil(M / 32)); 256 threads.  One CTA: 32 latents of one head
// over the token range of split blockIdx.x, in tiles of 32 tokens.
//   DEC: e = exp(s - lse3_t), g = Z_m . dY_t, ds = e (g - delta_t);
//        acc0 += e dY_t (-> dZ), acc1 += ds K_t (-> dQ_dyn, decode part)
//   ENC: e = exp(s - L_m), g = G_m . V_t, ds = e (g - c_m);
//        acc1 += ds K_t (-> dQ_dyn routing part with L = lse2, G = dZ, c = c2,
//        or d_seeds with the seeds, L = lse1, G = dQ_dyn, c = c1)
// Partials go to part[(bh * S + split) * M + m][d] (acc1) and, for DEC, the
// same place in the second block (acc0).
enum BwdMode { kBwdDec = 0, kBwdEncRouting = 1, kBwdEncSeed = 2 };

template <int D, typename T, int MODE>
__global__ void __launch_bounds__(kBwdThreads) latent_grad_kernel(const BwdArgs a) {
  extern __shared__ float sm[];
  constexpr int P = D + 1;
  float* sQ = sm;                          // logits' latent side  [32][P]
  float* sG = sQ + kBwdChunk * P;          // gradient latent side [32][P]
  float* sK = sG + kBwdChunk * P;          // K tile
  float* sX = sK + kBwdChunk * P;          // dY (DEC) or V (ENC) tile
  float* sE = sX + kBwdChunk * P;          // [32 latents][33]
  float* sS = sE + kBwdChunk * (kBwdChunk + 1);
  float* sTok = sS + kBwdChunk * (kBwdChunk + 1);  // [2][32] per-token stats (DEC)
  const int split = blockIdx.x, bh = blockIdx.y;
  const int m0 = blockIdx.z * kBwdChunk;
  const int h = bh % a.H;
  const size_t lat_base = static_cast<size_t>(bh) * a.M;
  const size_t tok_base = static_cast<size_t>(bh) * a.N;

  if constexpr (MODE == kBwdDec) {
    load_rows<D>(sQ, static_cast<const T*>(a.Qd) + lat_base * D, m0, a.M);
    load_rows<D>(sG, static_cast<const T*>(a.Z) + lat_base * D, m0, a.M);
  } else if constexpr (MODE == kBwdEncRouting) {
    load_rows<D>(sQ, static_cast<const T*>(a.Qd) + lat_base * D, m0, a.M);
    load_rows<D>(sG, a.dZ + lat_base * D, m0, a.M);
  } else {
    load_rows<D>(sQ, static_cast<const T*>(a.seeds) + static_cast<size_t>(h) * a.M * D, m0, a.M);
    load_rows<D>(sG, a.dQd + lat_base * D, m0, a.M);
  }
  // phase-1 mapping: lane = token of the tile, rows warp + 8 j
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float Lm[4], cm[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int m = m0 + warp + 8 * j;
    Lm[j] = 0.f;
    cm[j] = 0.f;
    if constexpr (MODE != kBwdDec) {
      if (m < a.M) {
        Lm[j] = (MODE == kBwdEncRouting ? a.lse2 : a.lse1)[lat_base + m];
        cm[j] = (MODE == kBwdEncRouting ? a.c2 : a.c1)[lat_base + m];
      }
    }
  }
  // phase-2 mapping: channel d, latent rows r0 + k * RS
  constexpr int RS = kBwdThreads / D;          // rows per pass
  constexpr int RK = kBwdChunk / RS;           // rows per thread
  const int pd = threadIdx.x % D, pr = threadIdx.x / D;
  float acc0[RK], acc1[RK];
#pragma unroll
  for (int k = 0; k < RK; ++k) acc0[k] = acc1[k] = 0.f;

  const long long tok0 = static_cast<long long>(split) * a.N / a.S;
  const long long tok1 = static_cast<long long>(split + 1) * a.N / a.S;
  const T* Kh = static_cast<const T*>(a.K) + tok_base * D;
  const T* Xh = static_cast<const T*>(MODE == kBwdDec ? a.dY : a.V) + tok_base * D;
  for (long long t0 = tok0; t0 < tok1; t0 += kBwdChunk) {
    __syncthreads();
    load_rows<D>(sK, Kh, t0, tok1);
    load_rows<D>(sX, Xh, t0, tok1);
    if constexpr (MODE == kBwdDec) {
      if (threadIdx.x < kBwdChunk) {
        const long long t = t0 + threadIdx.x;
        sTok[threadIdx.x] = t < tok1 ? a.lse3[tok_base + t] : INFINITY;  // exp(s - inf) = 0
        sTok[kBwdChunk + threadIdx.x] = t < tok1 ? a.delta[tok_base + t] : 0.f;
      }
    }
    __syncthreads();
    const bool tok_live = t0 + lane < tok1;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = warp + 8 * j;
      const bool live = tok_live && m0 + r < a.M;
      float e = 0.f, ds = 0.f;
      if (live) {
        const float s = dot_rows<D>(sQ + r * P, sK + lane * P);
        const float g = dot_rows<D>(sG + r * P, sX + lane * P);
        if constexpr (MODE == kBwdDec) {
          e = expf(s - sTok[lane]);
          ds = e * (g - sTok[kBwdChunk + lane]);
        } else {
          e = expf(s - Lm[j]);
          ds = e * (g - cm[j]);
        }
      }
      sE[r * (kBwdChunk + 1) + lane] = e;
      sS[r * (kBwdChunk + 1) + lane] = ds;
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kBwdChunk; ++t) {
      const float kv = sK[t * P + pd];
      const float xv = sX[t * P + pd];
#pragma unroll
      for (int k = 0; k < RK; ++k) {
        const int r = pr + k * RS;
        acc1[k] = fmaf(sS[r * (kBwdChunk + 1) + t], kv, acc1[k]);
        if constexpr (MODE == kBwdDec) acc0[k] = fmaf(sE[r * (kBwdChunk + 1) + t], xv, acc0[k]);
      }
    }
  }
  const size_t row0 = (static_cast<size_t>(bh) * a.S + split) * a.M;
#pragma unroll
  for (int k = 0; k < RK; ++k) {
    const int m = m0 + pr + k * RS;
    if (m < a.M) {
      a.part[(row0 + m) * D + pd] = acc1[k];
      if constexpr (MODE == kBwdDec) a.part[a.part_stride + (row0 + m) * D + pd] = acc0[k];
    }
  }
}

// ---------------------------------------------------------------- reductions
// grid (ceil(M / 8), heads); 256 threads = 8 warps, one latent row per warp,
// lanes over the D channels.  Sums the partials of one output row:
//   DEC     (heads = BH): dZ = sum_s part2, dQ_dyn = sum_s part1,
//                         c2 = dZ . Z
//   ROUTING (heads = BH): dQ_dyn += sum_s part1, c1 = dQ_dyn . Q_dyn
//   SEED    (heads = H):  d_seeds[h] = sum_b sum_s part1   (stored as T)
// STAGE 0 does it in one go.  A token-sharded backward splits it around the
// sum over ranks: STAGE 1 writes this rank's sums to the exchange buffer
// (DEC: dZ then dQ_dyn), and after the caller has summed that buffer over the
// ranks, STAGE 2 takes the sums from it and does the rest.
enum BwdStage { kStageFused = 0, kStageLocal = 1, kStageFinish = 2 };

template <int D, typename T, int MODE, int STAGE>
__global__ void __launch_bounds__(kBwdThreads) grad_reduce_kernel(const BwdArgs a, int B) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * 8 + warp;
  const int head = blockIdx.y;
  if (m >= a.M) return;  // whole warp
  float dot = 0.f;
  for (int d = lane; d < D; d += 32) {
    float v = 0.f, v0 = 0.f;
    if constexpr (MODE == kBwdEncSeed) {
      const size_t o = (static_cast<size_t>(head) * a.M + m) * D + d;
      if constexpr (STAGE == kStageFinish) {
        v = a.exch[o];
      } else {
        for (int b = 0; b < B; ++b) {
          const size_t row0 = (static_cast<size_t>(b * a.H + head) * a.S) * a.M + m;
          for (int s = 0; s < a.S; ++s) v += a.part[(row0 + static_cast<size_t>(s) * a.M) * D + d];
        }
      }
      if constexpr (STAGE == kStageLocal)
        a.exch[o] = v;
      else
        st_from_f32(static_cast<T*>(a.d_seeds) + o, v);
    } else {
      const size_t o = (static_cast<size_t>(head) * a.M + m) * D + d;
      const size_t L = static_cast<size_t>(gridDim.y) * a.M * D;  // one [BH][M][D] block
      if constexpr (STAGE == kStageFinish) {
        if constexpr (MODE == kBwdDec) {
          v0 = a.exch[o];
          v = a.exch[L + o];
        } else {
          v = a.exch[o];
        }
      } else {
        const size_t row0 = static_cast<size_t>(head) * a.S * a.M + m;
        for (int s = 0; s < a.S; ++s) {
          const size_t i = (row0 + static_cast<size_t>(s) * a.M) * D + d;
          v += a.part[i];
          if constexpr (MODE == kBwdDec) v0 += a.part[a.part_stride + i];
        }
      }
      if constexpr (STAGE == kStageLocal) {
        if constexpr (MODE == kBwdDec) {
          a.exch[o] = v0;
          a.exch[L + o] = v;
        } else {
          a.exch[o] = v;
        }
        continue;
      }
      // With bf16 copies (the tensor-core kernels take dZ V^T and dQ_dyn V^T
      // from them), the row terms c2 = dZ . Z and c1 = dQ_dyn . Q_dyn use the
      // same rounded values: then each softmax-gradient row still sums to
      // zero (sum_n A (dA - c) = 0 when c = sum_n A dA), and the rounding of
      // dZ and dQ_dyn is not amplified by the cancellation between dA and c.
      if constexpr (MODE == kBwdDec) {
        a.dQd[o] = v;
        a.dZ[o] = v0;
        if (a.dZ16) {
          const __nv_bfloat16 r = __float2bfloat16_rn(v0);
          a.dZ16[o] = r;
          v0 = __bfloat162float(r);
        }
        dot = fmaf(v0, ld_f32(static_cast<const T*>(a.Z) + o), dot);
      } else {
        v += a.dQd[o];
        a.dQd[o] = v;
        if (a.dQd16) {
          const __nv_bfloat16 r = __float2bfloat16_rn(v);
          a.dQd16[o] = r;
          v = __bfloat162float(r);
        }
        dot = fmaf(v, ld_f32(static_cast<const T*>(a.Qd) + o), dot);
      }
    }
  }
  if constexpr (MODE != kBwdEncSeed && STAGE != kStageLocal) {
    dot = warp_sum(dot);
    if (lane == 0) (MODE == kBwdDec ? a.c2 : a.c1)[static_cast<size_t>(head) * a.M + m] = dot;
  }
}

// ---------------------------------------------------------------- token rows
// grid (ceil(N / 32), BH); 256 threads.  One CTA: 32 tokens of one head; the
// latents in chunks of 32.  Phase 1 (lane = latent, rows warp + 8 j = tokens):
//   s = K_t . Q_dyn_m (S3 = S2^T), s1 = K_t . Q~_m
//   ds3 = exp(s - lse3_t) (dY_t . Z_m - delta_t)
//   a2 = exp(s - lse2_m),  ds2 = a2 (V_t . dZ_m - c2_m)
//   a1 = exp(s1 - lse1_m), ds1 = a1 (V_t . dQ_dyn_m - c1_m)
// Phase 2 (thread = channel d, token rows): dK += (ds3 + ds2) Q_dyn_m + ds1 Q~_m,
//   dV += a2 dZ_m + a1 dQ_dyn_m.
template <int D, typename T>
__global__ void __launch_bounds__(kBwdThreads) token_grad_kernel(const BwdArgs a) {
  extern __shared__ float sm[];
  constexpr int P = D + 1;
  constexpr int W = kBwdChunk + 1;
  float* sK = sm;
  float* sV = sK + kBwdChunk * P;
  float* sG = sV + kBwdChunk * P;    // dY
  float* sQ = sG + kBwdChunk * P;    // Q_dyn chunk
  float* sZ = sQ + kBwdChunk * P;
  float* sdZ = sZ + kBwdChunk * P;
  float* sS1 = sdZ + kBwdChunk * P;  // seeds chunk
  float* sdQ = sS1 + kBwdChunk * P;  // dQ_dyn chunk
  float* wQ = sdQ + kBwdChunk * P;   // [32 tokens][33] coefficient of Q_dyn_m in dK
  float* wS = wQ + kBwdChunk * W;    // of Q~_m in dK
  float* wZ = wS + kBwdChunk * W;    // of dZ_m in dV
  float* wD = wZ + kBwdChunk * W;    // of dQ_dyn_m in dV
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y, h = bh % a.H;
  const long long t0 = static_cast<long long>(blockIdx.x) * kBwdChunk;
  const size_t tok_base = static_cast<size_t>(bh) * a.N;
  const size_t lat_base = static_cast<size_t>(bh) * a.M;
  load_rows<D>(sK, static_cast<const T*>(a.K) + tok_base * D, t0, a.N);
  load_rows<D>(sV, static_cast<const T*>(a.V) + tok_base * D, t0, a.N);
  load_rows<D>(sG, static_cast<const T*>(a.dY) + tok_base * D, t0, a.N);
  float l3[4], dl[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const long long t = t0 + warp + 8 * j;
    l3[j] = t < a.N ? a.lse3[tok_base + t] : 0.f;
    dl[j] = t < a.N ? a.delta[tok_base + t] : 0.f;
  }
  constexpr int RS = kBwdThreads / D;
  constexpr int RK = kBwdChunk / RS;
  const int pd = threadIdx.x % D, pr = threadIdx.x / D;
  float gk[RK], gv[RK];
#pragma unroll
  for (int k = 0; k < RK; ++k) gk[k] = gv[k] = 0.f;

  for (int m0 = 0; m0 < a.M; m0 += kBwdChunk) {
    __syncthreads();
    load_rows<D>(sQ, static_cast<const T*>(a.Qd) + lat_base * D, m0, a.M);
    load_rows<D>(sZ, static_cast<const T*>(a.Z) + lat_base * D, m0, a.M);
    load_rows<D>(sdZ, a.dZ + lat_base * D, m0, a.M);
    load_rows<D>(sS1, static_cast<const T*>(a.seeds) + static_cast<size_t>(h) * a.M * D, m0, a.M);
    load_rows<D>(sdQ, a.dQd + lat_base * D, m0, a.M);
    __syncthreads();
    const int m = m0 + lane;
    const bool lat_live = m < a.M;
    const float L1 = lat_live ? a.lse1[lat_base + m] : 0.f;
    const float L2 = lat_live ? a.lse2[lat_base + m] : 0.f;
    const float C1 = lat_live ? a.c1[lat_base + m] : 0.f;
    const float C2 = lat_live ? a.c2[lat_base + m] : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = warp + 8 * j;
      float q = 0.f, sd = 0.f, z = 0.f, dq = 0.f;
      if (lat_live && t0 + t < a.N) {
        const float* kt = sK + t * P;
        const float* vt = sV + t * P;
        const float s = dot_rows<D>(kt, sQ + lane * P);
        const float s1 = dot_rows<D>(kt, sS1 + lane * P);
        const float ds3 = expf(s - l3[j]) * (dot_rows<D>(sG + t * P, sZ + lane * P) - dl[j]);
        const float a2 = expf(s - L2);
        const float a1 = expf(s1 - L1);
        q = ds3 + a2 * (dot_rows<D>(vt, sdZ + lane * P) - C2);
        sd = a1 * (dot_rows<D>(vt, sdQ + lane * P) - C1);
        z = a2;
        dq = a1;
      }
      wQ[t * W + lane] = q;
      wS[t * W + lane] = sd;
      wZ[t * W + lane] = z;
      wD[t * W + lane] = dq;
    }
    __syncthreads();
#pragma unroll 4
    for (int mm = 0; mm < kBwdChunk; ++mm) {
      const float qv = sQ[mm * P + pd], sv = sS1[mm * P + pd];
      const float zv = sdZ[mm * P + pd], dv = sdQ[mm * P + pd];
#pragma unroll
      for (int k = 0; k < RK; ++k) {
        const int t = pr + k * RS;
        gk[k] = fmaf(wQ[t * W + mm], qv, fmaf(wS[t * W + mm], sv, gk[k]));
        gv[k] = fmaf(wZ[t * W + mm], zv, fmaf(wD[t * W + mm], dv, gv[k]));
      }
    }
  }
#pragma unroll
  for (int k = 0; k < RK; ++k) {
    const long long t = t0 + pr + k * RS;
    if (t < a.N) {
      st_from_f32(static_cast<T*>(a.dK) + (tok_base + t) * D + pd, gk[k]);
      st_from_f32(static_cast<T*>(a.dV) + (tok_base + t) * D + pd, gv[k]);
    }
  }
}

template <int D>
constexpr int bwd_smem_token_stats() {
  return 4 * kBwdChunk * (D + 1) * 4;
}
template <int D>
constexpr int bwd_smem_latent() {
  return (4 * kBwdChunk * (D + 1) + 2 * kBwdChunk * (kBwdChunk + 1) + 2 * kBwdChunk) * 4;
}
template <int D>
constexpr int bwd_smem_token_grad() {
  return (8 * kBwdChunk * (D + 1) + 4 * kBwdChunk * (kBwdChunk + 1)) * 4;
}

}  // namespace flare
