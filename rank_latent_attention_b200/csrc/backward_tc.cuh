// Token side of the FLARE++ backward on the tensor cores: dK and dV.
//
// For a tile of 128 tokens t of one head and the latents m in chunks of 32
// (the same formulas as token_grad_kernel, see backward_simt.cuh):
//   logits (tcgen05, bf16 in, fp32 in TMEM; 128 x 32 each, K = D)
//     S3  = K_t Q_dyn^T     dP3 = dY_t Z^T     dA2 = V_t dZ^T
//     S1  = K_t Q~^T        dA1 = V_t dQ_dyn^T
//   weights (one thread per token row, written back to TMEM as bf16)
//     wQ = exp(S3 - lse3_t)(dP3 - delta_t) + exp(S3 - lse2_m)(dA2 - c2_m)
//     wS = exp(S1 - lse1_m)(dA1 - c1_m)
//     wZ = exp(S3 - lse2_m)          wD = exp(S1 - lse1_m)
//   accumulate (tcgen05, A = weights from TMEM, B = latent rows MN-major)
//     dK += wQ Q_dyn + wS Q~         dV += wZ dZ + wD dQ_dyn
// dZ and dQ_dyn enter the MMAs as bf16 copies of their fp32 sums.
//
// One CTA per (token range, head); the five [M][D] latent matrices of the
// head stay in shared memory for the whole range (TMA, loaded once), the
// token tiles K, dY, V come in by TMA per tile.  Warps 0-3 own TMEM lanes
// 0-127 (one token row per thread); warp 4 issues the TMA loads and the MMAs.
// The schedule is serial: logits, weights, accumulation, chunk after chunk.
//
// TMEM columns: S3 [0,32) dP3 [32,64) dA2 [64,96) S1 [96,128) dA1 [128,160),
// weights wQ [160,176) wS [176,192) wZ [192,208) wD [208,224) (bf16 pairs),
// dK [224, 224+D), dV [224+D, 224+2D).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx_sm100.cuh"

namespace flare {

constexpr int kBtcTile = 128;  // tokens per tile (MMA M)
constexpr int kBtcChunk = 32;  // latents per chunk (logit MMA N, accumulate MMA K)

struct BwdTcArgs {
  int N, M, H, splits, tiles;
  const float* lse1;  // [BH][M] natural log
  const float* lse2;
  const float* c1;
  const float* c2;
  const float* lse3;  // [BH][N]
  const float* delta;
  __nv_bfloat16* dK;  // [BH][N][D]
  __nv_bfloat16* dV;
  int* status;
  unsigned long long wait_ns;
};

template <int D>
struct BtcCfg {
  using G = TileGeom<D>;
  static constexpr int kThreads = 160;
  static constexpr int kIssuerWarp = 4;
  static constexpr int kMPad = 256;  // latent rows reserved per matrix (M <= 256)
  static constexpr int kLatBytes = G::bytes(kMPad);
  static constexpr int kTokBytes = G::bytes(kBtcTile);
  static constexpr int kOffLat = 0;                        // Q_dyn, Z, dZ, Q~, dQ_dyn
  static constexpr int kOffTok = 5 * kLatBytes;            // K, dY, V
  static constexpr int kOffStats = kOffTok + 3 * kTokBytes;  // L1, L2, C1, C2 [kMPad]
  static constexpr int kOffBars = kOffStats + 4 * kMPad * 4;
  static constexpr int kNumBars = 8;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kColW = 160;
  static constexpr uint32_t kColDK = 224;
  static constexpr uint32_t kColDV = 224 + D;
  static_assert(kColDV + D <= 512, "TMEM budget");
  static constexpr uint32_t kIdescLogit = ptx::idesc_bf16(kBtcTile, kBtcChunk, 0, 0);
  static constexpr uint32_t kIdescAcc = ptx::idesc_bf16(kBtcTile, D, 0, 1);
};

enum { kSiteBwdIssuer = 7, kSiteBwdWeights = 8 };

template <int D>
__global__ void __launch_bounds__(BtcCfg<D>::kThreads, 1)
    token_grad_tc_kernel(const __grid_constant__ CUtensorMap tmQd, const __grid_constant__ CUtensorMap tmZ,
                         const __grid_constant__ CUtensorMap tmdZ, const __grid_constant__ CUtensorMap tmS,
                         const __grid_constant__ CUtensorMap tmdQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmdY, const __grid_constant__ CUtensorMap tmV,
                         const BwdTcArgs args) {
  using C = BtcCfg<D>;
  using G = typename C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* bar_lat = bars + 0;   // latent matrices landed
  uint64_t* bar_tok = bars + 1;   // token tile landed
  uint64_t* bar_S = bars + 2;     // logits of a chunk computed
  uint64_t* bar_W = bars + 3;     // weights of a chunk stored (4 warps)
  uint64_t* bar_acc = bars + 4;   // last accumulation of a tile done
  uint64_t* bar_free = bars + 5;  // dK, dV of a tile read out (4 warps)
  uint64_t* drain = bars + 6;
  float* sL1 = reinterpret_cast<float*>(smem + C::kOffStats);
  float* sL2 = sL1 + C::kMPad;
  float* sC1 = sL2 + C::kMPad;
  float* sC2 = sC1 + C::kMPad;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, bh = blockIdx.y, h = bh % args.H;
  const int tile0 = static_cast<int>((static_cast<long long>(split) * args.tiles) / args.splits);
  const int tile1 = static_cast<int>((static_cast<long long>(split + 1) * args.tiles) / args.splits);
  const int T = tile1 - tile0;
  const int nC = (args.M + kBtcChunk - 1) / kBtcChunk;
  const size_t lat_base = static_cast<size_t>(bh) * args.M;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_lat, 1);
    ptx::mbar_init(bar_tok, 1);
    ptx::mbar_init(bar_S, 1);
    ptx::mbar_init(bar_W, 4);
    ptx::mbar_init(bar_acc, 1);
    ptx::mbar_init(bar_free, 4);
    ptx::mbar_init(drain, 32);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  // per-latent statistics, log2 domain for the exponentials; padded latents
  // get +inf (their encode weights are then exactly 0)
  constexpr float kL2e = 1.4426950408889634f;
  for (int m = threadIdx.x; m < C::kMPad; m += blockDim.x) {
    const bool live = m < args.M;
    sL1[m] = live ? args.lse1[lat_base + m] * kL2e : INFINITY;
    sL2[m] = live ? args.lse2[lat_base + m] * kL2e : INFINITY;
    sC1[m] = live ? args.c1[lat_base + m] : 0.f;
    sC2[m] = live ? args.c2[lat_base + m] : 0.f;
  }
  if (warp == C::kIssuerWarp) {
    ptx::tmem_alloc(s_tmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = ptx::smem_u32(smem);

  if (warp == C::kIssuerWarp) {
    // ---------------------------------------------------------------- loads + MMAs
    const uint32_t aLat = sbase + C::kOffLat;  // matrix j at aLat + j * kLatBytes
    const uint32_t aTok = sbase + C::kOffTok;  // K, dY, V
    const int boxes = (args.M + 63) / 64;
    bool ok = true;
    int tok_issued = -1;
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(bar_lat, 5 * boxes * 64 * D * 2);
      const CUtensorMap* maps[5] = {&tmQd, &tmZ, &tmdZ, &tmS, &tmdQ};
      for (int j = 0; j < 5; ++j) {
        const int plane = j == 3 ? h : bh;
        for (int bx = 0; bx < boxes; ++bx)
          ptx::tma_load_3d(smem + C::kOffLat + j * C::kLatBytes + bx * 64 * G::kRowBytes, maps[j], bar_lat, 0,
                           bx * 64, plane);
      }
    }
    __syncwarp();
    int kc = 0;  // chunks issued so far (parity of bar_S / bar_W)
    for (int i = 0; ok && i < T; ++i) {
      if (i > 0) ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, (i - 1) & 1, s_abort, args.wait_ns));
      if (!ok) break;
      if (ptx::elect_one()) {
        const int tok = (tile0 + i) * kBtcTile;
        ptx::mbar_arrive_expect_tx(bar_tok, 3 * C::kTokBytes);
        ptx::tma_load_3d(smem + C::kOffTok, &tmK, bar_tok, 0, tok, bh);
        ptx::tma_load_3d(smem + C::kOffTok + C::kTokBytes, &tmdY, bar_tok, 0, tok, bh);
        ptx::tma_load_3d(smem + C::kOffTok + 2 * C::kTokBytes, &tmV, bar_tok, 0, tok, bh);
      }
      __syncwarp();
      tok_issued = i;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_tok, i & 1, s_abort, args.wait_ns) &&
                                       (i > 0 || ptx::mbar_wait(bar_lat, 0, s_abort, args.wait_ns)));
      for (int c = 0; ok && c < nC; ++c, ++kc) {
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          const uint32_t lat_off = static_cast<uint32_t>(c * kBtcChunk * G::kRowBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t dKt = G::kmajor(aTok, kBtcTile, k);
            const uint64_t ddY = G::kmajor(aTok + C::kTokBytes, kBtcTile, k);
            const uint64_t dVt = G::kmajor(aTok + 2 * C::kTokBytes, kBtcTile, k);
            const uint32_t acc = k > 0 ? 1u : 0u;
            ptx::mma_ss(tmem + 0, dKt, G::kmajor(aLat + 0 * C::kLatBytes + lat_off, C::kMPad, k), C::kIdescLogit, acc);
            ptx::mma_ss(tmem + 32, ddY, G::kmajor(aLat + 1 * C::kLatBytes + lat_off, C::kMPad, k), C::kIdescLogit, acc);
            ptx::mma_ss(tmem + 64, dVt, G::kmajor(aLat + 2 * C::kLatBytes + lat_off, C::kMPad, k), C::kIdescLogit, acc);
            ptx::mma_ss(tmem + 96, dKt, G::kmajor(aLat + 3 * C::kLatBytes + lat_off, C::kMPad, k), C::kIdescLogit, acc);
            ptx::mma_ss(tmem + 128, dVt, G::kmajor(aLat + 4 * C::kLatBytes + lat_off, C::kMPad, k), C::kIdescLogit,
                        acc);
          }
          ptx::mma_commit(bar_S);
        }
        __syncwarp();
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_W, kc & 1, s_abort, args.wait_ns) &&
                                         (c > 0 || i == 0 || ptx::mbar_wait(bar_free, (i - 1) & 1, s_abort, args.wait_ns)));
        if (!ok) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          const uint32_t lat_off = static_cast<uint32_t>(c * kBtcChunk * G::kRowBytes);
#pragma unroll
          for (int kk = 0; kk < kBtcChunk / 16; ++kk) {
            const uint32_t first = (c == 0 && kk == 0) ? 0u : 1u;
            auto mn = [&](int j) { return G::mnmajor(aLat + j * C::kLatBytes + lat_off, C::kMPad, kk); };
            ptx::mma_ts(tmem + C::kColDK, tmem + C::kColW + 0 + kk * 8, mn(0), C::kIdescAcc, first);
            ptx::mma_ts(tmem + C::kColDK, tmem + C::kColW + 16 + kk * 8, mn(3), C::kIdescAcc, 1u);
            ptx::mma_ts(tmem + C::kColDV, tmem + C::kColW + 32 + kk * 8, mn(2), C::kIdescAcc, first);
            ptx::mma_ts(tmem + C::kColDV, tmem + C::kColW + 48 + kk * 8, mn(4), C::kIdescAcc, 1u);
          }
          if (c == nC - 1) ptx::mma_commit(bar_acc);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (lane == 0) record_error(args.status, kErrTimeout, kSiteBwdIssuer);
      *s_abort = 1;
    }
    // every MMA and every load issued completes before the CTA releases TMEM
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
    if (tok_issued >= 0) ptx::mbar_wait_drain(bar_tok, tok_issued & 1);
    ptx::mbar_wait_drain(bar_lat, 0);
  } else {
    // ---------------------------------------------------------------- weights
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t trow = tmem + lane_off;
    const size_t tok_base = static_cast<size_t>(bh) * args.N;
    bool ok = true;
    int kc = 0;
    for (int i = 0; ok && i < T; ++i) {
      const long long n = static_cast<long long>(tile0 + i) * kBtcTile + warp * 32 + lane;
      const bool live_tok = n < args.N;
      const float L3 = live_tok ? args.lse3[tok_base + n] * kL2e : 0.f;
      const float dl = live_tok ? args.delta[tok_base + n] : 0.f;
      for (int c = 0; c < nC; ++c, ++kc) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_S, kc & 1, s_abort, args.wait_ns));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float s3[16], dp[16], da2[16], s1[16], da1[16];
          ptx::tmem_ld16(trow + 0 + hh * 16, s3);
          ptx::tmem_ld16(trow + 32 + hh * 16, dp);
          ptx::tmem_ld16(trow + 64 + hh * 16, da2);
          ptx::tmem_ld16(trow + 96 + hh * 16, s1);
          ptx::tmem_ld16(trow + 128 + hh * 16, da1);
          ptx::tmem_wait_ld();
          uint32_t wq[8], ws[8], wz[8], wd[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            float q[2], sd[2], z[2], dq[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int j = 2 * u + e;
              const int m = c * kBtcChunk + hh * 16 + j;
              const float p3 = m < args.M ? ptx::ex2(fmaf(s3[j], kL2e, -L3)) : 0.f;
              const float a2 = ptx::ex2(fmaf(s3[j], kL2e, -sL2[m]));
              const float a1 = ptx::ex2(fmaf(s1[j], kL2e, -sL1[m]));
              q[e] = fmaf(p3, dp[j] - dl, a2 * (da2[j] - sC2[m]));
              sd[e] = a1 * (da1[j] - sC1[m]);
              z[e] = a2;
              dq[e] = a1;
            }
            wq[u] = ptx::pack_bf16(q[0], q[1]);
            ws[u] = ptx::pack_bf16(sd[0], sd[1]);
            wz[u] = ptx::pack_bf16(z[0], z[1]);
            wd[u] = ptx::pack_bf16(dq[0], dq[1]);
          }
          ptx::tmem_st8(trow + C::kColW + 0 + hh * 8, wq);
          ptx::tmem_st8(trow + C::kColW + 16 + hh * 8, ws);
          ptx::tmem_st8(trow + C::kColW + 32 + hh * 8, wz);
          ptx::tmem_st8(trow + C::kColW + 48 + hh * 8, wd);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_W);
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, i & 1, s_abort, args.wait_ns));
      if (!ok) break;
      ptx::tc_fence_after();
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* dst = (which == 0 ? args.dK : args.dV) + (tok_base + (live_tok ? n : 0)) * D;
        const uint32_t col = which == 0 ? C::kColDK : C::kColDV;
#pragma unroll
        for (int d0 = 0; d0 < D; d0 += 16) {
          float v[16];
          ptx::tmem_ld16(trow + col + d0, v);
          ptx::tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) pk[u] = ptx::pack_bf16(v[2 * u], v[2 * u + 1]);
          if (live_tok) {
            uint4* o = reinterpret_cast<uint4*>(dst + d0);
            o[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            o[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_free);
    }
    if (!ok) {
      if (lane == 0) record_error(args.status, kErrTimeout, kSiteBwdWeights);
      *s_abort = 1;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kIssuerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace flare
