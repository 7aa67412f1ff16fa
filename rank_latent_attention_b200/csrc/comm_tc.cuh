// Communication matrix of the latent routing on tcgen05 tensor cores, in one
// pass over the tokens.
//
//   C = W_enc W_dec  (M x M per head),  W_enc = softmax_N(Q K^T),
//                                         W_dec = softmax_M(K Q^T)
// ("FLARE: Fast Low-rank Attention Routing Engine" review page, sections
// "Матрица коммуникации низкого ранга" and "Спектральный анализ").  Both
// weights are functions of the same logits s_nm = k_n . q_m:
//   W_enc[m][n] = exp(s_nm - L2_m),  L2_m = log sum_n exp(s_nm)  (per latent)
//   W_dec[n][m] = exp(s_nm - L3_n),  L3_n = log sum_m exp(s_nm)  (per token)
// With L2 known (the log-sum-exp an encode's merge already produces), C is a
// plain sum over tokens of outer products, C = sum_n W_enc[:, n] W_dec[n, :],
// which needs no online rescaling: each token tile adds E^T P to C, with
// E[n][m] = W_enc[m][n] and P[n][m'] = W_dec[n][m'] both computed from the
// tile's logits by one thread per token (L3 is the thread's own row).
//
// Work of one CTA: one (b, h), one 128-latent half hm of C's rows, and a
// contiguous run of 128-token tiles.
//   warps 0-15 one token row per thread, four warps per TMEM lane quarter
//              (column quarter cq: latents [cq MP / 4, +MP / 4) of the row)
//   warp 16    TMA producer: Q once, K tiles into an NS ring; TMEM allocator
//   warp 17    tcgen05.mma issuer
// Per tile: S = K_t Q^T (128 x MP fp32, TMEM [0, MP)); the rows load S and
// free it (the issuer starts the next tile's S at once), exchange their
// quarter-row max and sum, and write P (all MP columns) and E (the columns in
// half hm) as fp16 into shared memory, in the MN-major layout with tokens as
// the reduction dimension; then C_hm += E^T P (M = 128, N = MP, K = 128
// tokens; C in TMEM [256, 256 + MP) fp32).  E is taken first, from the raw
// logits, into one of two E buffers; P then replaces the logits in
// registers and goes into the single P buffer once the previous tile's MMA
// has read it.  A tile's exponentials (the binding work, up to 3/2 MP per
// token) run while that MMA runs.
// Both weights lie in [0, 1], so fp16 holds them to 2^-11 relative (8x finer
// than bf16); E is stored as E 2^12, which keeps the typical encode weight
// (about 1/N) out of fp16's subnormal range, and the partials are scaled
// back by 2^-12 (exact).  The C MMA is kind::f16 with fp16 operands.
// Epilogue: C_hm of the CTA's token run into the partial block
// C_part[bh][split][m][m'] (fp32), summed over splits by comm_reduce_kernel.
#pragma once

#include <cuda_bf16.h>

#include <type_traits>

#include "common.cuh"

namespace flare {

constexpr int kSiteCommProducer = 7;
constexpr int kSiteCommMma = 8;
constexpr int kSiteCommRows = 9;

struct CommArgs {
  int N, M, H, q_batched;
  int splits, tiles;      // 128-token tiles per head
  const float* lse2;      // [BH][M] natural-log log-sum-exp over tokens of each latent's logits
  float* C_part;          // [BH][splits][M][M]
  int* status;
  unsigned long long wait_ns;
};

template <int D, int MP, int NS>
struct CommCfg {
  using G = TileGeom<D>;
  static_assert(D <= 64, "one column block per row");
  static_assert(MP == 128 || MP == 256, "padded latent count");
  static constexpr int kHalves = MP / kLatRows;  // 128-latent halves of C's rows
  static constexpr int kColGroups = 4;           // row warps per TMEM lane quarter
  static constexpr int kCols = MP / kColGroups;  // S columns per row warp
  static constexpr int kRowWarps = 4 * kColGroups;
  static constexpr int kProducerWarp = kRowWarps;
  static constexpr int kIssuerWarp = kRowWarps + 1;
  static constexpr int kThreads = 32 * (kRowWarps + 2);
  static constexpr int kLatBytes = G::bytes(MP);     // Q [MP][D]
  static constexpr int kTileBytes = G::bytes(kTileN);  // K tile [128][D]
  // E [128 tokens][128 latents] and P [128 tokens][MP latents], bf16, MN-major:
  // column blocks of 64 latents, each [128 tokens][64] with 128-byte rows
  static constexpr int kBlockBytes = kTileN * 128;
  static constexpr int kEBytes = 2 * kBlockBytes;  // E of 128 latents
  static constexpr int kOffQ = 0;
  static constexpr int kOffStages = kLatBytes;
  static constexpr int kOffE = kOffStages + NS * kTileBytes;  // two E buffers
  static constexpr int kOffP = kOffE + 2 * kEBytes;
  static constexpr int kOffBars = kOffP + (MP / 64) * kBlockBytes;
  // full[NS], empty[NS], q_full, S_full, S_free, AB_full, P_free, E_free[2], drain
  static constexpr int kNumBars = 2 * NS + 8;
  static constexpr int kOffBias = kOffBars + 8 * kNumBars;  // float [MP]: 12 - lse2 log2e (-inf past M)
  static constexpr int kOffX = kOffBias + MP * 4;  // float [2 use][kColGroups][128]: partial row max, sum
  static constexpr int kOffMisc = kOffX + 2 * kColGroups * 128 * 4;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColC = 256;
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16(kTileN, MP, 0, 0);
  static constexpr uint32_t kIdescC = ptx::idesc_f16(kLatRows, MP, 1, 1);  // fp16 A and B, both MN-major
  static constexpr float kEScaleLog2 = 12.f;  // E is stored as E 2^12
};

// Byte offset of the 16-byte chunk c (8 latents) of token row r in an
// MN-major block [128][64] with 128-byte rows, as the tensor core reads it
// with the 128-byte swizzle.
__device__ __forceinline__ uint32_t comm_chunk_offset(int r, int c) {
  return static_cast<uint32_t>(r * 128 + ((c ^ (r & 7)) << 4));
}

template <int D, int MP, int NS>
__global__ void __launch_bounds__(CommCfg<D, MP, NS>::kThreads, 1)
    comm_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                   const CommArgs args) {
  using C = CommCfg<D, MP, NS>;
  using G = typename C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_full = bars + 2 * NS;
  uint64_t* S_full = q_full + 1;
  uint64_t* S_free = q_full + 2;
  uint64_t* AB_full = q_full + 3;
  uint64_t* P_free = q_full + 4;  // the MMA of the last tile has read P
  uint64_t* E_free = q_full + 5;  // [buffer]: the MMA of the last tile that used it has read it
  uint64_t* drain = q_full + 7;
  float* s_bias = reinterpret_cast<float*>(smem + C::kOffBias);
  float* s_x = reinterpret_cast<float*>(smem + C::kOffX);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int hm = blockIdx.y;  // 128-latent half of C's rows
  const int bh = blockIdx.z;
  const int tile0 = static_cast<int>((static_cast<long long>(split) * args.tiles) / args.splits);
  const int tile1 = static_cast<int>((static_cast<long long>(split + 1) * args.tiles) / args.splits);
  const int T = tile1 - tile0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(S_full, 1);
    ptx::mbar_init(S_free, C::kRowWarps);  // one arrival per row warp
    ptx::mbar_init(AB_full, C::kRowWarps);
    ptx::mbar_init(P_free, 1);
    ptx::mbar_init(&E_free[0], 1);
    ptx::mbar_init(&E_free[1], 1);
    ptx::mbar_init(drain, 32);  // one commit per lane of the issuer warp
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  // the exponent bias of each latent's encode weight, 2^12 / exp(lse2_m) in
  // log2 units (-inf past M, whose weights are then 0)
  for (int m = threadIdx.x; m < MP; m += C::kThreads)
    s_bias[m] = m < args.M ? C::kEScaleLog2 - args.lse2[static_cast<size_t>(bh) * args.M + m] * kLog2e : -INFINITY;
  if (warp == C::kProducerWarp) {
    ptx::tmem_alloc(s_tmem, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = ptx::smem_u32(smem);

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmQ);
      const int qidx = args.q_batched ? bh : bh % args.H;
      ptx::mbar_arrive_expect_tx(q_full, C::kLatBytes);
      for (int h = 0; h < MP / kLatRows; ++h)
        ptx::tma_load_3d(smem + C::kOffQ + h * kLatRows * G::kRowBytes, &tmQ, q_full, 0, h * kLatRows, qidx);
      const uint64_t pol = ptx::policy_evict_first();
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % NS;
        if (t >= NS && !ptx::mbar_wait(&empty[st], ((t / NS) - 1) & 1, s_abort, args.wait_ns)) {
          record_error(args.status, kErrTimeout, kSiteCommProducer);
          *s_abort = 1;
          break;
        }
        ptx::mbar_arrive_expect_tx(&full[st], C::kTileBytes);
        ptx::tma_load_3d_hint(smem + C::kOffStages + st * C::kTileBytes, &tmK, &full[st], 0, (tile0 + t) * kTileN,
                              bh, pol);
        issued = t + 1;
      }
      ptx::mbar_wait_drain(q_full, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        ptx::mbar_wait_drain(&full[t % NS], (t / NS) & 1);
    }
  } else if (warp == C::kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dK0 = G::kmajor(sbase + C::kOffStages, kTileN, 0);
    const uint64_t dQ = G::kmajor(sbase + C::kOffQ, MP, 0);
    const uint64_t dE = ptx::smem_desc(sbase + C::kOffE, C::kBlockBytes, 1024, 2);
    const uint64_t dP = ptx::smem_desc(sbase + C::kOffP, C::kBlockBytes, 1024, 2);
    auto issue_qk = [&](int t) {
      const uint64_t dK = dK0 + static_cast<uint32_t>((t % NS) * (C::kTileBytes >> 4));
#pragma unroll
      for (int k = 0; k < D / 16; ++k)
        ptx::mma_ss(tmem, dK + G::kmajor_step(kTileN, k), dQ + G::kmajor_step(MP, k), C::kIdescQK, k > 0 ? 1u : 0u);
      ptx::mma_commit(S_full);
      ptx::mma_commit(&empty[t % NS]);
    };
    auto wait_stage = [&](int t) -> bool {
      return ptx::mbar_wait(&full[t % NS], (t / NS) & 1, s_abort, args.wait_ns);
    };
    bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(q_full, 0, s_abort, args.wait_ns));
    if (ok && T > 0) {
      ok = __all_sync(0xffffffffu, wait_stage(0));
      if (ok) {
        ptx::tc_fence_after();
        if (ptx::elect_one()) issue_qk(0);
        __syncwarp();
      }
    }
    for (int t = 0; ok && t < T; ++t) {
      // S(t) loaded by every row: the next tile's logits may overwrite it
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(S_free, t & 1, s_abort, args.wait_ns) &&
                                       (t + 1 >= T || wait_stage(t + 1)));
      if (!ok) break;
      ptx::tc_fence_after();
      if (t + 1 < T && ptx::elect_one()) issue_qk(t + 1);
      __syncwarp();
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(AB_full, t & 1, s_abort, args.wait_ns));
      if (!ok) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        // C_hm += E^T P over the tile's 128 tokens, K steps of 16 token rows
        const uint64_t dEt = dE + static_cast<uint32_t>(((t & 1) * C::kEBytes) >> 4);
#pragma unroll
        for (int k = 0; k < kTileN / 16; ++k)
          ptx::mma_ss(tmem + C::kColC, dEt + static_cast<uint32_t>((k * 16 * 128) >> 4),
                      dP + static_cast<uint32_t>((k * 16 * 128) >> 4), C::kIdescC, (t > 0 || k > 0) ? 1u : 0u);
        ptx::mma_commit(P_free);
        ptx::mma_commit(&E_free[t & 1]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      record_error(args.status, kErrTimeout, kSiteCommMma);
      *s_abort = 1;
    }
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
  } else {
    // ------------------------------------------------------------ token rows
    // Each warp takes runs of 32 latents, one run in each 128-latent half
    // (latents [32 cq, +32) and, with MP = 256, [128 + 32 cq, +32)), so every
    // warp forms the same share of E (its run in half hm) and of P.
    const int q = warp & 3;       // TMEM lane quarter
    const int cq = warp >> 2;     // which run of each half
    const int r = q * 32 + lane;  // token row of the tile
    const uint32_t tRow = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int bar_id = 1 + q;     // the four warps of this lane quarter
    constexpr int kG = C::kColGroups;
    constexpr int kRuns = C::kCols / 32;  // runs of 32 latents per thread
    float* xm = s_x;              // [cq][128]
    float* xs = s_x + kG * 128;
    auto run_col = [&](int run) { return run * kLatRows + 32 * cq; };  // first latent of a run
    const int e_run = hm;  // the run that lies in half hm (MP = 128: hm = 0, one run)
    const uint64_t kL2 = ptx::f2(kLog2e, kLog2e);
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(S_full, t & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float x[C::kCols];
#pragma unroll
      for (int run = 0; run < kRuns; ++run) ptx::tmem_ld32(tRow + run_col(run), x + 32 * run);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(S_free);
      // a row past N (a ragged last tile) contributes nothing: its logits
      // are set to 0 (finite) and its weights zeroed below
      const bool valid = (tile0 + t) * kTileN + r < args.N;
      const bool all_valid = __all_sync(0xffffffffu, valid);
      // latents past M take no part (M is a multiple of 16; only a run that
      // crosses M needs the mask)
#pragma unroll
      for (int run = 0; run < kRuns; ++run) {
        if (run_col(run) + 32 > args.M) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (run_col(run) + j >= args.M) x[32 * run + j] = -INFINITY;
        }
      }
      float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < C::kCols; j += 8) {
        pm[0] = ptx::max3(pm[0], x[j], x[j + 1]);
        pm[1] = ptx::max3(pm[1], x[j + 2], x[j + 3]);
        pm[2] = ptx::max3(pm[2], x[j + 4], x[j + 5]);
        pm[3] = ptx::max3(pm[3], x[j + 6], x[j + 7]);
      }
      xm[cq * 128 + r] = fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
      asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
      const float rowmax = fmaxf(fmaxf(xm[r], xm[128 + r]), fmaxf(xm[256 + r], xm[384 + r])) * kLog2e;
      // E = 2^(s log2e + 12 - lse2_m) from the raw logits, for this thread's
      // run in half hm, into E buffer t % 2 once the MMA of tile t - 2 has
      // read it (s_bias[m] = 12 - lse2_m log2e, -inf past M)
      if (t >= 2 &&
          !__all_sync(0xffffffffu, ptx::mbar_wait(&E_free[t & 1], ((t - 2) >> 1) & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      {
        uint8_t* eb = smem + C::kOffE + (t & 1) * C::kEBytes;
        // the run index is a compile-time constant in each branch, so x
        // stays in registers
        auto form_e = [&](auto run_c) {
          constexpr int run = decltype(run_c)::value;
          const float2* bias = reinterpret_cast<const float2*>(s_bias + run_col(run));
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t e[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int j = 8 * c + 2 * u;
              const float2 b = bias[j / 2];
              const uint64_t a = ptx::fma2(ptx::f2(x[32 * run + j], x[32 * run + j + 1]), kL2, ptx::f2(b.x, b.y));
              float a0, a1;
              ptx::f2_split(a, a0, a1);
              float e0 = ptx::ex2(a0), e1 = ptx::ex2(a1);
              if (!all_valid && !valid) e0 = e1 = 0.f;
              e[u] = ptx::pack_f16(e0, e1);
            }
            const int col = 32 * cq + 8 * c;  // latent within half hm
            *reinterpret_cast<uint4*>(eb + (col / 64) * C::kBlockBytes + comm_chunk_offset(r, (col % 64) / 8)) =
                make_uint4(e[0], e[1], e[2], e[3]);
          }
        };
        if (kRuns == 1 || e_run == 0)
          form_e(std::integral_constant<int, 0>{});
        else
          form_e(std::integral_constant<int, kRuns - 1>{});
      }
      // decode weights of this row: 2^(s log2e - rowmax), normalised below
      const uint64_t nr = ptx::f2(-rowmax, -rowmax);
      uint64_t ps[2] = {0ull, 0ull};
#pragma unroll
      for (int j = 0; j < C::kCols; j += 2) {
        float a0, a1;
        ptx::f2_split(ptx::fma2(ptx::f2(x[j], x[j + 1]), kL2, nr), a0, a1);
        x[j] = ptx::ex2(a0);
        x[j + 1] = ptx::ex2(a1);
        ps[(j >> 1) & 1] = ptx::add2(ps[(j >> 1) & 1], ptx::f2(x[j], x[j + 1]));
      }
      float s0, s1, s2, s3;
      ptx::f2_split(ps[0], s0, s1);
      ptx::f2_split(ps[1], s2, s3);
      xs[cq * 128 + r] = (s0 + s1) + (s2 + s3);
      asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
      const float inv = valid ? 1.f / ((xs[r] + xs[128 + r]) + (xs[256 + r] + xs[384 + r])) : 0.f;
      const uint64_t inv2 = ptx::f2(inv, inv);
      // the previous tile's MMA has read the P buffer
      if (t > 0 && !__all_sync(0xffffffffu, ptx::mbar_wait(P_free, (t - 1) & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      // P: chunks of 8 latents into the column blocks of 64
#pragma unroll
      for (int c = 0; c < C::kCols / 8; ++c) {
        const int col = run_col(c / 4) + 8 * (c % 4);  // first latent of the chunk
        uint32_t v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float p0, p1;
          ptx::f2_split(ptx::mul2(ptx::f2(x[8 * c + 2 * u], x[8 * c + 2 * u + 1]), inv2), p0, p1);
          v[u] = ptx::pack_f16(p0, p1);
        }
        *reinterpret_cast<uint4*>(smem + C::kOffP + (col / 64) * C::kBlockBytes + comm_chunk_offset(r, (col % 64) / 8)) =
            make_uint4(v[0], v[1], v[2], v[3]);
      }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(AB_full);
    }
    if (!ok) {
      record_error(args.status, kErrTimeout, kSiteCommRows);
      *s_abort = 1;
    }
    // ---------------------------------------------------------- epilogue
    // C_hm row (latent hm 128 + 32 q + lane) of this CTA's tokens, columns
    // [cq MP / 4, +MP / 4), into the split's partial block
    if (ok && T > 0 && __all_sync(0xffffffffu, ptx::mbar_wait(P_free, (T - 1) & 1, s_abort, args.wait_ns))) {
      ptx::tc_fence_after();
      const int m = hm * kLatRows + r;
      const int c0 = cq * C::kCols;  // this warp's contiguous share of C's columns
      float* dst = args.C_part + ((static_cast<size_t>(bh) * args.splits + split) * args.M + m) * args.M;
#pragma unroll
      for (int k = 0; k < C::kCols / 32; ++k) {
        float cv[32];
        ptx::tmem_ld32(tmem + C::kColC + (static_cast<uint32_t>(q * 32) << 16) + cq * C::kCols + 32 * k, cv);
        ptx::tmem_wait_ld();
        if (m < args.M) {
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const int col = c0 + 32 * k + j;
            constexpr float kUnscale = 1.f / 4096.f;  // 2^-12: E was stored as E 2^12
            if (col < args.M)
              *reinterpret_cast<float4*>(dst + col) =
                  make_float4(cv[j] * kUnscale, cv[j + 1] * kUnscale, cv[j + 2] * kUnscale, cv[j + 3] * kUnscale);
          }
        }
      }
    } else if (ok && T > 0) {
      record_error(args.status, kErrTimeout, kSiteCommRows);
      *s_abort = 1;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kProducerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// C[bh][m][m'] = sum over the splits of C_part (fp32 or bf16 out); one
// thread per element.
template <typename OutT>
__global__ void __launch_bounds__(256) comm_reduce_kernel(const float* __restrict__ C_part, OutT* __restrict__ C,
                                                          int M, int splits) {
  const size_t mm = static_cast<size_t>(M) * M;
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= mm) return;
  const int bh = blockIdx.y;
  const float* src = C_part + static_cast<size_t>(bh) * splits * mm + idx;
  float acc = 0.f;
  for (int s = 0; s < splits; ++s) acc += src[s * mm];
  if constexpr (std::is_same<OutT, float>::value)
    C[static_cast<size_t>(bh) * mm + idx] = acc;
  else
    C[static_cast<size_t>(bh) * mm + idx] = __float2bfloat16_rn(acc);
}

}  // namespace flare
