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
// token tiles K, dY, V come in by TMA per tile.  Warps 0-15 turn logits into
// weights, four per TMEM lane quarter (one token row per thread, 8 of a
// chunk's 32 latents per warp).  Two issuer warps: warp 16 issues the TMA
// loads and the logit MMAs, warp 17 the accumulation MMAs.  A thread with
// MMAs in flight stalls on its next mbarrier wait until they complete, so
// with one issuer every wait (for weights, for a buffer, for the next token
// tile) also waited for the other kind of MMA; measured on one B200 the
// single issuer held a chunk to ~2,400 clocks where its MMAs take ~860.
// Logits run two chunks ahead in two TMEM buffers: the logits of chunk g + 2
// go into chunk g's buffer as soon as every row has read chunk g, while the
// rows turn it into weights.  The weights have a TMEM region of their own,
// single-buffered: the rows store chunk g + 1's once the accumulation of
// chunk g has read chunk g's.  The token buffer is single: the next tile's
// K, dY, V are loaded as soon as the logits of this tile's last chunk are
// done, and only the logits issuer waits for them to land.
//
// TMEM columns: logit buffer b at 160 b: S3 [0,32) S1 [32,64) dA2 [64,96)
// dA1 [96,128) dP3 [128,160) (S3 | S1 and dA2 | dA1 are one MMA each);
// weights (bf16 pairs) at 320: wQ, wS, wZ, wD 16 columns each, K step kk of
// the accumulation (latents [16 kk, +16) of the chunk) at 8 kk of each;
// dK [384, 384+D), dV [384+D, 384+2D).
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
  static constexpr int kRowWarps = 16;  // four per TMEM lane quarter
  static constexpr int kIssuerWarp = 16;  // logits and loads; warp 17: accumulation
  static constexpr int kThreads = 32 * 18;
  static constexpr int kLatPerWarp = kBtcChunk / 4;  // latents of a chunk per row warp
  static constexpr int kMPad = 256;  // latent rows reserved per matrix (M <= 256)
  static constexpr int kLatBytes = G::bytes(kMPad);
  // Latent rows in shared memory, chunk by chunk: block c holds the 32 rows
  // of chunk c of Q_dyn, Q~, dZ, dQ_dyn, Z in that order, so that (Q_dyn; Q~)
  // and (dZ; dQ_dyn) are 64-row B operands: one MMA each against K_t and V_t.
  static constexpr int kChunkRows = 5 * kBtcChunk;
  __host__ __device__ static constexpr uint32_t lat_row(int c, int pos) {
    return static_cast<uint32_t>((c * 5 + pos) * kBtcChunk);
  }
  static constexpr int kTokBytes = G::bytes(kBtcTile);
  static constexpr int kOffLat = 0;                        // Q_dyn, Z, dZ, Q~, dQ_dyn
  static constexpr int kOffTok = 5 * kLatBytes;            // K, dY, V
  static constexpr int kOffStats = kOffTok + 3 * kTokBytes;  // float4 {L1, L2, c1, c2} [kMPad]
  static constexpr int kOffBars = kOffStats + 4 * kMPad * 4;
  static constexpr int kNumBars = 12;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kBufCols = 160;
  static constexpr uint32_t kColW = 2 * kBufCols;
  // which: 0 wQ, 1 wS, 2 wZ, 3 wD; K step kk covers latents [16 kk, +16) of the chunk
  __host__ __device__ static constexpr uint32_t w_col(int which, int kk) { return kColW + which * 16 + kk * 8; }
  static constexpr uint32_t kColDK = kColW + 64;
  static constexpr uint32_t kColDV = kColDK + D;
  static_assert(kColDV + D <= 512, "TMEM budget");
  static constexpr uint32_t kIdescLogit = ptx::idesc_bf16(kBtcTile, kBtcChunk, 0, 0);
  static constexpr uint32_t kIdescLogit2 = ptx::idesc_bf16(kBtcTile, 2 * kBtcChunk, 0, 0);
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
  uint64_t* bar_tok = bars + 1;   // a token tile landed (once per tile)
  uint64_t* bar_S = bars + 2;     // [2] logits of a chunk computed, per buffer
  uint64_t* bar_R = bars + 4;     // [2] logits of a chunk read by every row warp (16), per buffer
  uint64_t* bar_W = bars + 6;     // weights of a chunk stored (16)
  uint64_t* bar_accd = bars + 7;  // accumulation of a chunk done (its weights read)
  uint64_t* bar_acc = bars + 8;   // last accumulation of a tile done
  uint64_t* bar_free = bars + 9;  // dK, dV of a tile read out (16)
  uint64_t* drain = bars + 10;
  float4* sStat = reinterpret_cast<float4*>(smem + C::kOffStats);  // per latent {L1, L2, c1, c2}
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
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&bar_S[b], 1);
      ptx::mbar_init(&bar_R[b], C::kRowWarps);
    }
    ptx::mbar_init(bar_W, C::kRowWarps);
    ptx::mbar_init(bar_accd, 1);
    ptx::mbar_init(bar_acc, 1);
    ptx::mbar_init(bar_free, C::kRowWarps);
    ptx::mbar_init(drain, 64);  // one commit per lane of the two issuer warps
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  // per-latent statistics, log2 domain for the exponentials; padded latents
  // get +inf (their encode weights are then exactly 0)
  constexpr float kL2e = 1.4426950408889634f;
  for (int m = threadIdx.x; m < C::kMPad; m += blockDim.x) {
    const bool live = m < args.M;
    sStat[m] = live ? make_float4(args.lse1[lat_base + m] * kL2e, args.lse2[lat_base + m] * kL2e, args.c1[lat_base + m],
                                  args.c2[lat_base + m])
                    : make_float4(INFINITY, INFINITY, 0.f, 0.f);
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

  if (warp >= C::kIssuerWarp) {
    // ---------------------------------------------------------------- loads + MMAs
    // Each issuer warp runs its loop as a whole (waits are warp-wide); one
    // elected lane issues each batch of MMAs, loads and commits.
    const uint32_t aLat = sbase + C::kOffLat;  // matrix j at aLat + j * kLatBytes
    const uint32_t aTok = sbase + C::kOffTok;  // K, dY, V
    const int nG = T * nC;  // chunks of the CTA, in order; chunk g uses logit buffer g & 1
    bool ok = true;
    int tok_issued = -1;
    auto wait = [&](uint64_t* bar, int parity) -> bool {
      return __all_sync(0xffffffffu, ptx::mbar_wait(bar, parity, s_abort, args.wait_ns));
    };
    if (warp == C::kIssuerWarp) {
      // ------------------------------------------------ logits and loads
      if (ptx::elect_one()) {
        ptx::mbar_arrive_expect_tx(bar_lat, 5 * nC * kBtcChunk * D * 2);
        const CUtensorMap* maps[5] = {&tmQd, &tmS, &tmdZ, &tmdQ, &tmZ};  // block order
        for (int c = 0; c < nC; ++c)
          for (int j = 0; j < 5; ++j)
            ptx::tma_load_3d(smem + C::kOffLat + C::lat_row(c, j) * G::kRowBytes, maps[j], bar_lat, 0,
                             c * kBtcChunk, j == 1 ? h : bh);
      }
      __syncwarp();
      auto load_tokens = [&](int i) {
        if (ptx::elect_one()) {
          const int tok = (tile0 + i) * kBtcTile;
          ptx::mbar_arrive_expect_tx(bar_tok, 3 * C::kTokBytes);
          ptx::tma_load_3d(smem + C::kOffTok, &tmK, bar_tok, 0, tok, bh);
          ptx::tma_load_3d(smem + C::kOffTok + C::kTokBytes, &tmdY, bar_tok, 0, tok, bh);
          ptx::tma_load_3d(smem + C::kOffTok + 2 * C::kTokBytes, &tmV, bar_tok, 0, tok, bh);
        }
        __syncwarp();
        tok_issued = i;
      };
      if (nG > 0) {
        load_tokens(0);
        ok = wait(bar_tok, 0) && wait(bar_lat, 0);
      }
      // Operand descriptors built once: only the start-address field moves
      // between K steps, chunks and tensors, so each MMA adds a constant (the
      // issuer shares its SMSP with busy row warps; rebuilding 64-bit
      // descriptors per MMA made each batch several hundred clocks long).
      const uint64_t dTok = G::kmajor(aTok, kBtcTile, 0);  // K; dY and V kTokStep and 2 kTokStep on
      constexpr uint32_t kTokStep = static_cast<uint32_t>(C::kTokBytes) >> 4;
      const uint64_t dLat = G::kmajor(aLat, 2 * kBtcChunk, 0);
      for (int g = 0; ok && g < nG; ++g) {
        // a tile's first chunk: its tokens were loaded once the logits of the
        // tile before were done
        if (g % nC == 0 && g > 0 && !(ok = wait(bar_tok, (g / nC) & 1))) break;
        // the buffer of chunk g - 2 has been read by every row warp
        if (g >= 2 && !(ok = wait(&bar_R[g & 1], ((g - 2) >> 1) & 1))) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          const uint32_t buf = tmem + C::kBufCols * (g & 1);
          const int c = g % nC;
          auto lat = [&](int pos) { return dLat + ((C::lat_row(c, pos) * G::kRowBytes) >> 4); };
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t sk = G::kmajor_step(kBtcTile, k);
            const uint32_t acc = k > 0 ? 1u : 0u;
            ptx::mma_ss(buf + 0, dTok + sk, lat(0) + G::kmajor_step(2 * kBtcChunk, k), C::kIdescLogit2, acc);  // S3 | S1
            ptx::mma_ss(buf + 64, dTok + 2 * kTokStep + sk, lat(2) + G::kmajor_step(2 * kBtcChunk, k), C::kIdescLogit2,
                        acc);                                                                                 // dA2 | dA1
            ptx::mma_ss(buf + 128, dTok + kTokStep + sk, lat(4) + G::kmajor_step(kBtcChunk, k), C::kIdescLogit,
                        acc);                                                                                 // dP3
          }
          ptx::mma_commit(&bar_S[g & 1]);
        }
        __syncwarp();
        // the last chunk of a tile: once its logits are done, the token
        // buffer takes the next tile
        if (g + 1 < nG && (g + 1) % nC == 0) {
          if (!(ok = wait(&bar_S[g & 1], (g >> 1) & 1))) break;
          load_tokens((g + 1) / nC);
        }
      }
    } else {
      // ------------------------------------------------ accumulation
      const uint64_t dLatMN = G::mnmajor(aLat, C::kChunkRows, 0);  // built once, as the logits' descriptors
      for (int g = 0; ok && g < nG; ++g) {
        const int i = g / nC, c = g % nC;
        // the first chunk of a tile also waits for the previous tile's dK, dV
        // to be read out
        ok = wait(bar_W, g & 1) && (c > 0 || i == 0 || wait(bar_free, (i - 1) & 1));
        if (!ok) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBtcChunk / 16; ++kk) {
            const uint32_t first = (c == 0 && kk == 0) ? 0u : 1u;
            auto mn = [&](int pos) {
              return dLatMN + ((C::lat_row(c, pos) * G::kRowBytes) >> 4) + G::mnmajor_step(kk);
            };
            ptx::mma_ts(tmem + C::kColDK, tmem + C::w_col(0, kk), mn(0), C::kIdescAcc, first);  // wQ Q_dyn
            ptx::mma_ts(tmem + C::kColDK, tmem + C::w_col(1, kk), mn(1), C::kIdescAcc, 1u);     // wS Q~
            ptx::mma_ts(tmem + C::kColDV, tmem + C::w_col(2, kk), mn(2), C::kIdescAcc, first);  // wZ dZ
            ptx::mma_ts(tmem + C::kColDV, tmem + C::w_col(3, kk), mn(3), C::kIdescAcc, 1u);     // wD dQ_dyn
          }
          ptx::mma_commit(bar_accd);
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
    // (each lane of both issuer warps commits)
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
    if (tok_issued >= 0) ptx::mbar_wait_drain(bar_tok, tok_issued & 1);
    if (warp == C::kIssuerWarp) ptx::mbar_wait_drain(bar_lat, 0);
  } else {
    // ---------------------------------------------------------------- weights
    const int quarter = warp & 3, hq = warp >> 2;  // TMEM lanes 32 quarter.., latents 8 hq.. of a chunk
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t trow = tmem + lane_off;
    const size_t tok_base = static_cast<size_t>(bh) * args.N;
    // this warp's weights: 4 columns (8 latents as bf16 pairs) of K step hq / 2
    const uint32_t wcol = (hq >> 1) * 8 + (hq & 1) * 4;
    // Read-out of dK (warps hq 0-1) or dV (hq 2-3): columns [d_lo, d_lo + D / 2)
    // of this lane's row.  Each lane writes its own row, so a store touches 32
    // lines: 32-byte stores (when both outputs are 32-byte aligned; 16-column
    // groups of a row half then are too) halve the requests of 16-byte ones.
    constexpr int kHalfD = D / 2;
    constexpr int kGroupCols = kHalfD < 16 ? kHalfD : 16;
    const int which = hq >> 1, d_lo = (hq & 1) * kHalfD;
    const uint32_t col_out = (which == 0 ? C::kColDK : C::kColDV) + d_lo;
    __nv_bfloat16* const out = which == 0 ? args.dK : args.dV;
    const bool wide = kGroupCols == 16 &&
                      ((reinterpret_cast<uintptr_t>(args.dK) | reinterpret_cast<uintptr_t>(args.dV)) & 31u) == 0;
    auto row_of = [&](int i) { return static_cast<long long>(tile0 + i) * kBtcTile + quarter * 32 + lane; };
    // a tile's row statistics are loaded while the tile before is read out
    auto row_stats = [&](int i, float& L3, float& dl) {
      const long long n = row_of(i);
      const bool live = n < args.N;
      L3 = live ? args.lse3[tok_base + n] * kL2e : 0.f;
      dl = live ? args.delta[tok_base + n] : 0.f;
    };
    float L3n = 0.f, dln = 0.f;  // the next tile's row statistics, loaded a tile ahead
    if (T > 0) row_stats(0, L3n, dln);
    bool ok = true;
    int kc = 0;
    for (int i = 0; ok && i < T; ++i) {
      const long long n = row_of(i);
      const bool live_tok = n < args.N;
      const float L3 = L3n, dl = dln;
      for (int c = 0; c < nC; ++c, ++kc) {
        const int b = kc & 1;
        const uint32_t buf = trow + C::kBufCols * b + hq * C::kLatPerWarp;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&bar_S[b], (kc >> 1) & 1, s_abort, args.wait_ns));
        if (!ok) break;
        ptx::tc_fence_after();
        float s3[8], dp[8], da2[8], s1[8], da1[8];
        ptx::tmem_ld8(buf + 0, s3);
        ptx::tmem_ld8(buf + 32, s1);
        ptx::tmem_ld8(buf + 64, da2);
        ptx::tmem_ld8(buf + 96, da1);
        ptx::tmem_ld8(buf + 128, dp);
        ptx::tmem_wait_ld();
        // the buffer may take the logits of chunk kc + 2
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bar_R[b]);
        uint32_t wq[4], ws[4], wz[4], wd[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float q[2], sd[2], z[2], dq[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 2 * u + e;
            const int m = c * kBtcChunk + hq * C::kLatPerWarp + j;
            const float4 st = sStat[m];
            const float p3 = m < args.M ? ptx::ex2(fmaf(s3[j], kL2e, -L3)) : 0.f;
            const float a2 = ptx::ex2(fmaf(s3[j], kL2e, -st.y));
            const float a1 = ptx::ex2(fmaf(s1[j], kL2e, -st.x));
            q[e] = fmaf(p3, dp[j] - dl, a2 * (da2[j] - st.w));
            sd[e] = a1 * (da1[j] - st.z);
            z[e] = a2;
            dq[e] = a1;
          }
          wq[u] = ptx::pack_bf16(q[0], q[1]);
          ws[u] = ptx::pack_bf16(sd[0], sd[1]);
          wz[u] = ptx::pack_bf16(z[0], z[1]);
          wd[u] = ptx::pack_bf16(dq[0], dq[1]);
        }
        // the weights region is free once the accumulation of chunk kc - 1 has read it
        if (kc > 0) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_accd, (kc - 1) & 1, s_abort, args.wait_ns));
          if (!ok) break;
          ptx::tc_fence_after();
        }
        ptx::tmem_st4(trow + C::w_col(0, 0) + wcol, wq);
        ptx::tmem_st4(trow + C::w_col(1, 0) + wcol, ws);
        ptx::tmem_st4(trow + C::w_col(2, 0) + wcol, wz);
        ptx::tmem_st4(trow + C::w_col(3, 0) + wcol, wd);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_W);
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_acc, i & 1, s_abort, args.wait_ns));
      if (!ok) break;
      // the next tile's row statistics: their loads overlap the read-out
      if (i + 1 < T) row_stats(i + 1, L3n, dln);
      ptx::tc_fence_after();
      __nv_bfloat16* dst = out + (tok_base + (live_tok ? n : 0)) * D + d_lo;
#pragma unroll
      for (int d0 = 0; d0 < kHalfD; d0 += kGroupCols) {
        float v[kGroupCols];
        if constexpr (kGroupCols == 16) ptx::tmem_ld16(trow + col_out + d0, v); else ptx::tmem_ld8(trow + col_out + d0, v);
        ptx::tmem_wait_ld();
        uint32_t pk[kGroupCols / 2];
#pragma unroll
        for (int u = 0; u < kGroupCols / 2; ++u) pk[u] = ptx::pack_bf16(v[2 * u], v[2 * u + 1]);
        if (live_tok) {
          if constexpr (kGroupCols == 16) {
            if (wide) {
              ptx::st_global_v8(dst + d0, pk);
              continue;
            }
          }
          uint4* o = reinterpret_cast<uint4*>(dst + d0);
#pragma unroll
          for (int z = 0; z < kGroupCols / 8; ++z) o[z] = make_uint4(pk[4 * z], pk[4 * z + 1], pk[4 * z + 2], pk[4 * z + 3]);
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

// ---------------------------------------------------------------------------
// Latent side of the backward on the tensor cores: per 128 latents of one head
// (MMA rows) over a token range in tiles of 64 (MMA N of the logits):
//   DEC   S = Q_dyn K_t^T, G = Z dY_t^T   e = exp(S - lse3_t), w = e (G - delta_t)
//         dZ += e dY_t,  dQ_dyn += w K_t          (decode part of dQ_dyn)
//   ENC   S = A K_t^T,   G = B V_t^T      e = exp(S - lse_m),  w = e (G - c_m)
//         out += w K_t   with (A, B, lse, c, out) = (Q_dyn, dZ, lse2, c2, dQ_dyn)
//         for the routing encode, (Q~, dQ_dyn, lse1, c1, d_seeds) for the seed encode
// The partial sums of the CTA's token range go to the same [BH][S][M][D] fp32
// blocks as latent_grad_kernel's, summed by grad_reduce_kernel.
//
// Warps 0-3: one latent row per thread.  Warp 4: TMA (a ring of token
// stages) and MMAs.  TMEM: S [0,64), G [64,128); out0 [128, 128+D) (dZ, DEC
// only), out1 [128+D, 128+2D).  DEC writes e and w (bf16 pairs) over the first
// half of S and of G once read, so the next tile's logits wait for the
// accumulation.  ENC has no out0 and needs no e: w gets 32 columns of its own
// and the next tile's logits are issued as soon as the rows have read S and
// G, ahead of this tile's accumulation (a ring of four stages keeps the token
// loads ahead of the shorter period).
constexpr int kBltcTok = 64;

struct BltcArgs {
  int N, M, S, tiles;
  const float* lse_row;  // ENC: [BH][M] lse of the encode (natural log)
  const float* c_row;    // ENC: [BH][M]
  const float* lse3;     // DEC: [BH][N]
  const float* delta;    // DEC: [BH][N]
  float* part;           // [BH][S][M][D] (out1), out0 at part + part_stride
  long long part_stride;
  int* status;
  unsigned long long wait_ns;
};

template <int D, int MODE>
struct BltcCfg {
  using G = TileGeom<D>;
  static constexpr int kThreads = 160;
  static constexpr int kIssuerWarp = 4;
  static constexpr int kStages = MODE == 0 ? 2 : 4;
  static constexpr int kLatBytes = G::bytes(128);
  static constexpr int kTokBytes = G::bytes(kBltcTok);
  static constexpr int kOffLat = 0;                                  // A, B [128][D]
  static constexpr int kOffTok = 2 * kLatBytes;                      // stage s: K, X
  static constexpr int kOffStat = kOffTok + kStages * 2 * kTokBytes;  // [2 buffers][2][64] floats
  static constexpr int kOffBars = kOffStat + 2 * 2 * kBltcTok * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kColOut0 = 128;
  static constexpr uint32_t kColOut1 = 128 + D;
  static_assert(kColOut1 + D <= 256, "TMEM budget (256 columns per CTA)");
  // ENC: w (64 tokens as bf16 pairs) in the first 32 free columns
  static constexpr uint32_t kColW = kColOut1 + D + kBltcTok / 2 <= 256 ? kColOut1 + D : kColOut0;
  static_assert(kColW + kBltcTok / 2 <= 256 && (kColW >= kColOut1 + D || kColW + kBltcTok / 2 <= kColOut1),
                "ENC weight columns");
  static constexpr uint32_t kIdescLogit = ptx::idesc_bf16(128, kBltcTok, 0, 0);
  static constexpr uint32_t kIdescAcc = ptx::idesc_bf16(128, D, 0, 1);
};

enum { kSiteBwdLatIssuer = 9, kSiteBwdLatWeights = 10 };

template <int D, int MODE>
__global__ void __launch_bounds__(BltcCfg<D, MODE>::kThreads, 1)
    latent_grad_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                          const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmX,
                          const BltcArgs args, int a_per_batch_head, int H) {
  using C = BltcCfg<D, MODE>;
  using G = typename C::G;
  constexpr bool kDec = MODE == 0;
  constexpr int NS = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* bar_lat = bars + 0;
  uint64_t* full = bars + 1;        // [NS] token stage landed
  uint64_t* empty = bars + 1 + NS;  // [NS] token stage consumed by the accumulation MMAs
  uint64_t* bar_S = bars + 1 + 2 * NS;
  uint64_t* bar_W = bar_S + 1;
  uint64_t* bar_fin = bar_S + 2;
  uint64_t* drain = bar_S + 3;
  uint64_t* bar_R = bar_S + 4;     // ENC: the rows have read S and G
  uint64_t* bar_accd = bar_S + 5;  // ENC: the accumulation has read w
  static_assert(1 + 2 * NS + 6 <= C::kNumBars, "barrier slots");
  float* sTok = reinterpret_cast<float*>(smem + C::kOffStat);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, bh = blockIdx.y, m0 = blockIdx.z * 128;
  const int tile0 = static_cast<int>((static_cast<long long>(split) * args.tiles) / args.S);
  const int tile1 = static_cast<int>((static_cast<long long>(split + 1) * args.tiles) / args.S);
  const int T = tile1 - tile0;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_lat, 1);
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(bar_S, 1);
    ptx::mbar_init(bar_W, 4);
    ptx::mbar_init(bar_fin, 1);
    ptx::mbar_init(drain, 32);
    ptx::mbar_init(bar_R, 4);
    ptx::mbar_init(bar_accd, 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == C::kIssuerWarp) {
    ptx::tmem_alloc(s_tmem, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = ptx::smem_u32(smem);

  if (warp == C::kIssuerWarp) {
    // ---------------------------------------------------------------- loads + MMAs
    const int planeA = a_per_batch_head ? bh : bh % H;
    auto load_tile = [&](int i) {
      const int st = i % NS;
      const int tok = (tile0 + i) * kBltcTok;
      ptx::mbar_arrive_expect_tx(&full[st], 2 * C::kTokBytes);
      ptx::tma_load_3d(smem + C::kOffTok + st * 2 * C::kTokBytes, &tmK, &full[st], 0, tok, bh);
      ptx::tma_load_3d(smem + C::kOffTok + st * 2 * C::kTokBytes + C::kTokBytes, &tmX, &full[st], 0, tok, bh);
    };
    int loaded = 0;
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(bar_lat, 2 * C::kLatBytes);
      ptx::tma_load_3d(smem + C::kOffLat, &tmA, bar_lat, 0, m0, planeA);
      ptx::tma_load_3d(smem + C::kOffLat + C::kLatBytes, &tmB, bar_lat, 0, m0, bh);
      for (int i = 0; i < NS && i < T; ++i) load_tile(i);
    }
    __syncwarp();
    loaded = T < NS ? T : NS;
    bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_lat, 0, s_abort, args.wait_ns));
    // Operand descriptors built once: only the start-address field moves
    // between K steps and stages, so each MMA adds a constant (the issuer
    // shares its SMSP with busy row warps, and rebuilding 64-bit descriptors
    // per MMA made each batch of MMAs several hundred clocks long).
    const uint64_t dA = G::kmajor(sbase + C::kOffLat, 128, 0);
    const uint64_t dB = G::kmajor(sbase + C::kOffLat + C::kLatBytes, 128, 0);
    const uint64_t dK0 = G::kmajor(sbase + C::kOffTok, kBltcTok, 0);
    const uint64_t dKmn0 = G::mnmajor(sbase + C::kOffTok, kBltcTok, 0);
    constexpr uint32_t kStageStep = static_cast<uint32_t>(2 * C::kTokBytes) >> 4;
    constexpr uint32_t kXStep = static_cast<uint32_t>(C::kTokBytes) >> 4;
    // logits of tile i into S/G (stage i % NS holds its tokens)
    auto issue_logits = [&](int i) {
      const int st = i % NS;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t acc = k > 0 ? 1u : 0u;
          const uint32_t sa = G::kmajor_step(128, k), sk = st * kStageStep + G::kmajor_step(kBltcTok, k);
          ptx::mma_ss(tmem + 0, dA + sa, dK0 + sk, C::kIdescLogit, acc);
          ptx::mma_ss(tmem + 64, dB + sa, dK0 + kXStep + sk, C::kIdescLogit, acc);
        }
        ptx::mma_commit(bar_S);
      }
      __syncwarp();
    };
    if constexpr (kDec) {
      if (ok && T > 0) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&full[0], 0, s_abort, args.wait_ns));
        if (ok) issue_logits(0);
      }
      for (int i = 0; ok && i < T; ++i) {
        const int st = i & 1;
        // Every wait before the MMAs (a wait after them stalls until they
        // complete): the rows' weights of tile i, and the tokens of tile i + 1.
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_W, i & 1, s_abort, args.wait_ns) &&
                                         (i + 1 >= T || ptx::mbar_wait(&full[st ^ 1], ((i + 1) >> 1) & 1, s_abort,
                                                                       args.wait_ns)));
        if (!ok) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBltcTok / 16; ++kk) {
            const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
            const uint32_t sm = st * kStageStep + G::mnmajor_step(kk);
            ptx::mma_ts(tmem + C::kColOut0, tmem + 0 + kk * 8, dKmn0 + kXStep + sm, C::kIdescAcc, acc);
            ptx::mma_ts(tmem + C::kColOut1, tmem + 64 + kk * 8, dKmn0 + sm, C::kIdescAcc, acc);
          }
          ptx::mma_commit(&empty[st]);
          if (i == T - 1) ptx::mma_commit(bar_fin);
        }
        __syncwarp();
        // The next tile's logits overwrite S/G, whose e and w the accumulation
        // just issued reads: the tensor pipe runs MMAs in issue order, so they
        // are issued right behind it instead of after it completes and after
        // the stage refill below (which took ~430 clocks off every tile).
        if (i + 1 < T) issue_logits(i + 1);
        if (i + 2 < T) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(&empty[st], (i >> 1) & 1, s_abort, args.wait_ns));
          if (!ok) break;
          if (ptx::elect_one()) load_tile(i + 2);
          __syncwarp();
          loaded = i + 3;
        }
      }
    } else {
      // Tile i + 1's logits go out once the rows have read S and G of tile i
      // (and its tokens have landed), ahead of tile i's accumulation: the
      // rows then find the next logits done when they finish a tile.
      if (ok && T > 0) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&full[0], 0, s_abort, args.wait_ns));
        if (ok) issue_logits(0);
      }
      for (int i = 0; ok && i < T; ++i) {
        const int st = i % NS;
        if (i + 1 < T) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_R, i & 1, s_abort, args.wait_ns) &&
                                           ptx::mbar_wait(&full[(i + 1) % NS], ((i + 1) / NS) & 1, s_abort,
                                                          args.wait_ns));
          if (!ok) break;
          issue_logits(i + 1);
        }
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_W, i & 1, s_abort, args.wait_ns));
        if (!ok) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kBltcTok / 16; ++kk) {
            const uint32_t acc = (i > 0 || kk > 0) ? 1u : 0u;
            ptx::mma_ts(tmem + C::kColOut1, tmem + C::kColW + kk * 8, dKmn0 + st * kStageStep + G::mnmajor_step(kk),
                        C::kIdescAcc, acc);
          }
          ptx::mma_commit(&empty[st]);
          ptx::mma_commit(bar_accd);
          if (i == T - 1) ptx::mma_commit(bar_fin);
        }
        __syncwarp();
        if (i + NS < T) {
          ok = __all_sync(0xffffffffu, ptx::mbar_wait(&empty[st], (i / NS) & 1, s_abort, args.wait_ns));
          if (!ok) break;
          if (ptx::elect_one()) load_tile(i + NS);
          __syncwarp();
          loaded = i + NS + 1;
        }
      }
    }
    if (!ok) {
      if (lane == 0) record_error(args.status, kErrTimeout, kSiteBwdLatIssuer);
      *s_abort = 1;
    }
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
    for (int t = (loaded > NS ? loaded - NS : 0); t < loaded; ++t) ptx::mbar_wait_drain(&full[t % NS], (t / NS) & 1);
    ptx::mbar_wait_drain(bar_lat, 0);
  } else {
    // ---------------------------------------------------------------- weights
    constexpr float kL2e = 1.4426950408889634f;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int m = m0 + warp * 32 + lane;
    const bool live_m = m < args.M;
    const size_t lat_row = static_cast<size_t>(bh) * args.M + (live_m ? m : 0);
    float Lm = 0.f, cm = 0.f;
    if constexpr (!kDec) {
      Lm = live_m ? args.lse_row[lat_row] * kL2e : INFINITY;
      cm = live_m ? args.c_row[lat_row] : 0.f;
    }
    const size_t tok_base = static_cast<size_t>(bh) * args.N;
    // DEC: threads 0-63 hold the {lse3 (log2 domain), delta} of token j of
    // the next tile, loaded a tile ahead: their latency overlaps a tile's
    // exponentials instead of stalling every row warp at the barrier
    auto tok_stat = [&](int i) -> float2 {
      const long long t = static_cast<long long>(tile0 + i) * kBltcTok + threadIdx.x;
      return t < args.N ? make_float2(args.lse3[tok_base + t] * kL2e, args.delta[tok_base + t]) : make_float2(0.f, 0.f);
    };
    float2 next_stat = make_float2(0.f, 0.f);
    if (kDec && threadIdx.x < kBltcTok && T > 0) next_stat = tok_stat(0);
    bool ok = true;
    for (int i = 0; ok && i < T; ++i) {
      const long long t0 = static_cast<long long>(tile0 + i) * kBltcTok;
      const int live_cols = static_cast<int>(args.N - t0 < kBltcTok ? args.N - t0 : kBltcTok);
      float2* stat = reinterpret_cast<float2*>(sTok) + (i & 1) * kBltcTok;  // {lse3 log2 domain, delta}
      if constexpr (kDec) {
        // the tile's token statistics, shared by the 128 rows (buffers
        // alternate by tile parity; every row warp has finished tile i - 2
        // once all of them have passed tile i - 1's barrier)
        if (threadIdx.x < kBltcTok) {
          stat[threadIdx.x] = next_stat;
          if (i + 1 < T) next_stat = tok_stat(i + 1);
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
      }
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_S, i & 1, s_abort, args.wait_ns));
      if (!ok) break;
      ptx::tc_fence_after();
      // Token pairs as packed fp32 (f32x2): the exponent argument, g - c and
      // the product take one instruction per pair, with the same roundings
      // as the scalar fmaf / subtract / multiply.  Columns past the last
      // token (a ragged final tile only) give e = w = 0.
      const bool ragged = live_cols < kBltcTok;  // uniform
      const float4* stat4 = reinterpret_cast<const float4*>(stat);
      const uint64_t kL2e2 = ptx::f2(kL2e, kL2e);
      const uint64_t nL = ptx::f2(-Lm, -Lm), nc = ptx::f2(-cm, -cm);
      if constexpr (!kDec) {
        // All of S and G read at once (128 registers a thread): the rows
        // release S/G to the next tile's logits (bar_R) before computing, and
        // before the first store of w wait for the accumulation of tile i - 1,
        // which reads the same columns.
        float sv[4][16], gv[4][16];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          ptx::tmem_ld16(trow + 0 + 16 * p, sv[p]);
          ptx::tmem_ld16(trow + 64 + 16 * p, gv[p]);
        }
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_R);
        bool wok = true;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          uint32_t pw[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 16 * p + 2 * u;  // tokens j, j + 1
            const uint64_t a = ptx::fma2(ptx::f2(sv[p][2 * u], sv[p][2 * u + 1]), kL2e2, nL);
            const uint64_t b = ptx::add2(ptx::f2(gv[p][2 * u], gv[p][2 * u + 1]), nc);
            float a0, a1;
            ptx::f2_split(a, a0, a1);
            const uint64_t w = ptx::mul2(ptx::f2(ptx::ex2(a0), ptx::ex2(a1)), b);
            float w0, w1;
            ptx::f2_split(w, w0, w1);
            if (ragged) {
              w0 = j < live_cols ? w0 : 0.f;
              w1 = j + 1 < live_cols ? w1 : 0.f;
            }
            pw[u] = ptx::pack_bf16(w0, w1);
          }
          if (p == 0 && i > 0) {
            wok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_accd, (i - 1) & 1, s_abort, args.wait_ns));
            ptx::tc_fence_after();
          }
          ptx::tmem_st8(trow + C::kColW + 8 * p, pw);
        }
        if (!wok) {
          ok = false;
          break;
        }
      } else {
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float sv[16], gv[16];
          ptx::tmem_ld16(trow + 0 + 16 * p, sv);
          ptx::tmem_ld16(trow + 64 + 16 * p, gv);
          ptx::tmem_wait_ld();
          uint32_t pe[8], pw[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = 16 * p + 2 * u;  // tokens j, j + 1
            const float4 tj = stat4[j / 2];  // {lse3, delta} of tokens j and j + 1
            const uint64_t a = ptx::fma2(ptx::f2(sv[2 * u], sv[2 * u + 1]), kL2e2, ptx::f2(-tj.x, -tj.z));
            const uint64_t b = ptx::add2(ptx::f2(gv[2 * u], gv[2 * u + 1]), ptx::f2(-tj.y, -tj.w));
            float a0, a1;
            ptx::f2_split(a, a0, a1);
            const uint64_t e = ptx::f2(ptx::ex2(a0), ptx::ex2(a1));
            const uint64_t w = ptx::mul2(e, b);
            float e0, e1, w0, w1;
            ptx::f2_split(e, e0, e1);
            ptx::f2_split(w, w0, w1);
            if (ragged) {
              e0 = j < live_cols ? e0 : 0.f;
              w0 = j < live_cols ? w0 : 0.f;
              e1 = j + 1 < live_cols ? e1 : 0.f;
              w1 = j + 1 < live_cols ? w1 : 0.f;
            }
            pe[u] = ptx::pack_bf16(e0, e1);
            pw[u] = ptx::pack_bf16(w0, w1);
          }
          // over columns of S and G this thread has already read
          ptx::tmem_st8(trow + 0 + 8 * p, pe);
          ptx::tmem_st8(trow + 64 + 8 * p, pw);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar_W);
    }
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_fin, 0, s_abort, args.wait_ns));
      if (ok) {
        ptx::tc_fence_after();
        const size_t row = (static_cast<size_t>(bh) * args.S + split) * args.M + (live_m ? m : 0);
#pragma unroll
        for (int which = kDec ? 0 : 1; which < 2; ++which) {
          float* dst = args.part + (which == 0 ? args.part_stride : 0) + row * D;
          const uint32_t col = which == 0 ? C::kColOut0 : C::kColOut1;
#pragma unroll
          for (int d0 = 0; d0 < D; d0 += 16) {
            float v[16];
            ptx::tmem_ld16(trow + col + d0, v);
            ptx::tmem_wait_ld();
            if (live_m) {
              float4* o = reinterpret_cast<float4*>(dst + d0);
#pragma unroll
              for (int z = 0; z < 4; ++z) o[z] = make_float4(v[4 * z], v[4 * z + 1], v[4 * z + 2], v[4 * z + 3]);
            }
          }
        }
      }
    } else if (ok && live_m) {
      // no tokens in this split: its partial is zero
      const size_t row = (static_cast<size_t>(bh) * args.S + split) * args.M + m;
      for (int which = kDec ? 0 : 1; which < 2; ++which)
        for (int d = 0; d < D; ++d) args.part[(which == 0 ? args.part_stride : 0) + row * D + d] = 0.f;
    }
    if (!ok) {
      if (lane == 0) record_error(args.status, kErrTimeout, kSiteBwdLatWeights);
      *s_abort = 1;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kIssuerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// Per-token statistics of the decode on the tensor cores: for 128 tokens of
// one head (MMA rows) and the latents in chunks of 64,
//   S3 = K_t Q_dyn^T,  dP3 = dY_t Z^T      (tcgen05, fp32 in TMEM)
// and, online over the chunks (log2 domain), one thread per token:
//   lse3_t  = log-sum-exp over the latents of S3,
//   delta_t = sum_m softmax(S3)_m dP3_m    (= dY_t . Y_t).
// Q_dyn and Z of the head stay in shared memory; logits are double-buffered
// in TMEM (buffer b: S3 at 128 b, dP3 at 128 b + 64).
constexpr int kBstChunk = 64;

struct BstArgs {
  int N, M, splits, tiles;
  float* lse3;  // [BH][N]
  float* delta;
  int* status;
  unsigned long long wait_ns;
};

template <int D>
struct BstCfg {
  using G = TileGeom<D>;
  static constexpr int kThreads = 160;
  static constexpr int kIssuerWarp = 4;
  static constexpr int kLatBytes = G::bytes(256);
  static constexpr int kTokBytes = G::bytes(128);
  static constexpr int kOffLat = 0;                  // Q_dyn, Z [256][D]
  static constexpr int kOffTok = 2 * kLatBytes;      // K, dY [128][D]
  static constexpr int kOffBars = kOffTok + 2 * kTokBytes;
  static constexpr int kNumBars = 8;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kIdesc = ptx::idesc_bf16(128, kBstChunk, 0, 0);
};

enum { kSiteBwdStatIssuer = 11, kSiteBwdStatRows = 12 };

template <int D>
__global__ void __launch_bounds__(BstCfg<D>::kThreads, 1)
    token_stats_tc_kernel(const __grid_constant__ CUtensorMap tmQd, const __grid_constant__ CUtensorMap tmZ,
                          const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmdY,
                          const BstArgs args) {
  using C = BstCfg<D>;
  using G = typename C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* bar_lat = bars + 0;
  uint64_t* bar_tok = bars + 1;
  uint64_t* bar_S = bars + 2;    // [2] logits of a chunk in buffer b
  uint64_t* bar_rel = bars + 4;  // [2] buffer b read by the 4 row warps
  uint64_t* bar_tdone = bars + 6;  // every MMA of a tile done (token tiles free)
  uint64_t* drain = bars + 7;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int tile0 = static_cast<int>((static_cast<long long>(split) * args.tiles) / args.splits);
  const int tile1 = static_cast<int>((static_cast<long long>(split + 1) * args.tiles) / args.splits);
  const int T = tile1 - tile0;
  const int nC = (args.M + kBstChunk - 1) / kBstChunk;

  if (threadIdx.x == 0) {
    ptx::mbar_init(bar_lat, 1);
    ptx::mbar_init(bar_tok, 1);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&bar_S[b], 1);
      ptx::mbar_init(&bar_rel[b], 4);
    }
    ptx::mbar_init(bar_tdone, 1);
    ptx::mbar_init(drain, 32);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == C::kIssuerWarp) {
    ptx::tmem_alloc(s_tmem, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = ptx::smem_u32(smem);

  if (warp == C::kIssuerWarp) {
    const int boxes = (args.M + 63) / 64;
    if (ptx::elect_one()) {
      ptx::mbar_arrive_expect_tx(bar_lat, 2 * boxes * 64 * D * 2);
      for (int bx = 0; bx < boxes; ++bx) {
        ptx::tma_load_3d(smem + C::kOffLat + bx * 64 * G::kRowBytes, &tmQd, bar_lat, 0, bx * 64, bh);
        ptx::tma_load_3d(smem + C::kOffLat + C::kLatBytes + bx * 64 * G::kRowBytes, &tmZ, bar_lat, 0, bx * 64, bh);
      }
    }
    __syncwarp();
    bool ok = true;
    int tok_issued = -1;
    int kc = 0;  // chunks issued (buffer kc & 1, its (kc >> 1)-th use)
    const uint32_t aQ = sbase + C::kOffLat, aZ = aQ + C::kLatBytes;
    const uint32_t aK = sbase + C::kOffTok, adY = aK + C::kTokBytes;
    for (int i = 0; ok && i < T; ++i) {
      if (i > 0) ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_tdone, (i - 1) & 1, s_abort, args.wait_ns));
      if (!ok) break;
      if (ptx::elect_one()) {
        const int tok = (tile0 + i) * 128;
        ptx::mbar_arrive_expect_tx(bar_tok, 2 * C::kTokBytes);
        ptx::tma_load_3d(smem + C::kOffTok, &tmK, bar_tok, 0, tok, bh);
        ptx::tma_load_3d(smem + C::kOffTok + C::kTokBytes, &tmdY, bar_tok, 0, tok, bh);
      }
      __syncwarp();
      tok_issued = i;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(bar_tok, i & 1, s_abort, args.wait_ns) &&
                                       (i > 0 || ptx::mbar_wait(bar_lat, 0, s_abort, args.wait_ns)));
      for (int c = 0; ok && c < nC; ++c, ++kc) {
        const int b = kc & 1;
        // the buffer's previous chunk has been read by the row warps
        if (kc >= 2) ok = __all_sync(0xffffffffu, ptx::mbar_wait(&bar_rel[b], ((kc >> 1) - 1) & 1, s_abort, args.wait_ns));
        if (!ok) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          const uint32_t off = static_cast<uint32_t>(c * kBstChunk * G::kRowBytes);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t acc = k > 0 ? 1u : 0u;
            ptx::mma_ss(tmem + 128 * b, G::kmajor(aK, 128, k), G::kmajor(aQ + off, 256, k), C::kIdesc, acc);
            ptx::mma_ss(tmem + 128 * b + 64, G::kmajor(adY, 128, k), G::kmajor(aZ + off, 256, k), C::kIdesc, acc);
          }
          ptx::mma_commit(&bar_S[b]);
          if (c == nC - 1) ptx::mma_commit(bar_tdone);
        }
        __syncwarp();
      }
    }
    if (!ok) {
      if (lane == 0) record_error(args.status, kErrTimeout, kSiteBwdStatIssuer);
      *s_abort = 1;
    }
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
    if (tok_issued >= 0) ptx::mbar_wait_drain(bar_tok, tok_issued & 1);
    ptx::mbar_wait_drain(bar_lat, 0);
  } else {
    constexpr float kL2e = 1.4426950408889634f;
    constexpr float kLn2 = 0.6931471805599453f;
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const size_t tok_base = static_cast<size_t>(bh) * args.N;
    bool ok = true;
    int kc = 0;
    for (int i = 0; ok && i < T; ++i) {
      float mx = -INFINITY, l = 0.f, acc = 0.f;
      for (int c = 0; c < nC; ++c, ++kc) {
        const int b = kc & 1;
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&bar_S[b], (kc >> 1) & 1, s_abort, args.wait_ns));
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int p = 0; p < kBstChunk / 16; ++p) {
          float sv[16], gv[16];
          ptx::tmem_ld16(trow + 128 * b + 16 * p, sv);
          ptx::tmem_ld16(trow + 128 * b + 64 + 16 * p, gv);
          ptx::tmem_wait_ld();
          const int mbase = c * kBstChunk + 16 * p;
          float cm = -INFINITY;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            sv[j] = mbase + j < args.M ? sv[j] * kL2e : -INFINITY;
            cm = fmaxf(cm, sv[j]);
          }
          const float nm = fmaxf(mx, cm);
          if (nm > mx) {
            const float sc = mx == -INFINITY ? 0.f : ptx::ex2(mx - nm);
            l *= sc;
            acc *= sc;
            mx = nm;
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float e = ptx::ex2(sv[j] - mx);  // 0 for masked latents
            l += e;
            acc = fmaf(e, gv[j], acc);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bar_rel[b]);
      }
      if (!ok) break;
      const long long n = static_cast<long long>(tile0 + i) * 128 + warp * 32 + lane;
      if (n < args.N) {
        args.lse3[tok_base + n] = (mx + __log2f(l)) * kLn2;
        args.delta[tok_base + n] = acc / l;
      }
    }
    if (!ok) {
      if (lane == 0) record_error(args.status, kErrTimeout, kSiteBwdStatRows);
      *s_abort = 1;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kIssuerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
}

}  // namespace flare
