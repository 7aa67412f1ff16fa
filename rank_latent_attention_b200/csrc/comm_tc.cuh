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
  static constexpr int kOffL2 = kOffBars + 8 * kNumBars;  // float [MP]: lse2 in log2 units
  static constexpr int kOffX = kOffL2 + MP * 4;  // float [2 use][kColGroups][128]: partial row max, sum
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
  float* s_l2 = reinterpret_cast<float*>(smem + C::kOffL2);
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
  // lse2 of the head's latents in log2 units (0 past M: those rows are masked)
  for (int m = threadIdx.x; m < MP; m += C::kThreads)
    s_l2[m] = m < args.M ? args.lse2[static_cast<size_t>(bh) * args.M + m] * kLog2e : 0.f;
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
    const int q = warp & 3;       // TMEM lane quarter
    const int cq = warp >> 2;     // column quarter
    const int r = q * 32 + lane;  // token row of the tile
    const uint32_t tS = tmem + (static_cast<uint32_t>(q * 32) << 16) + cq * C::kCols;
    const int bar_id = 1 + q;     // the four warps of this lane quarter
    constexpr int kG = C::kColGroups;
    float* xm = s_x;              // [cq][128]
    float* xs = s_x + kG * 128;
    const int c0 = cq * C::kCols;  // first latent of this thread's columns
    // E columns: this thread's columns all lie in one 128-latent half
    const bool e_here = c0 / kLatRows == hm;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(S_full, t & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float x[C::kCols];
#pragma unroll
      for (int k = 0; k < C::kCols / 32; ++k) ptx::tmem_ld32(tS + 32 * k, x + 32 * k);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(S_free);
      const bool valid = (tile0 + t) * kTileN + r < args.N;
      // latents past M take no part (M is a multiple of 16)
#pragma unroll
      for (int j = 0; j < C::kCols; ++j)
        if (c0 + j >= args.M) x[j] = -INFINITY;
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < C::kCols; ++j) mx = fmaxf(mx, x[j]);
      xm[cq * 128 + r] = mx;
      asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
      const float rowmax = fmaxf(fmaxf(xm[r], xm[128 + r]), fmaxf(xm[256 + r], xm[384 + r])) * kLog2e;
      // E = 2^(s log2e - lse2_m) from the raw logits, for the latents of half
      // hm, into E buffer t % 2 once the MMA of tile t - 2 has read it
      if (e_here) {
        if (t >= 2 &&
            !__all_sync(0xffffffffu, ptx::mbar_wait(&E_free[t & 1], ((t - 2) >> 1) & 1, s_abort, args.wait_ns))) {
          ok = false;
          break;
        }
        uint8_t* eb = smem + C::kOffE + (t & 1) * C::kEBytes;
#pragma unroll
        for (int c = 0; c < C::kCols / 8; ++c) {
          uint32_t e[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = 8 * c + 2 * u;
            const float e0 = valid ? ptx::ex2(fmaf(x[j], kLog2e, C::kEScaleLog2 - s_l2[c0 + j])) : 0.f;
            const float e1 = valid ? ptx::ex2(fmaf(x[j + 1], kLog2e, C::kEScaleLog2 - s_l2[c0 + j + 1])) : 0.f;
            e[u] = ptx::pack_f16(e0, e1);
          }
          const int col = (c0 + 8 * c) - hm * kLatRows;  // latent within half hm
          *reinterpret_cast<uint4*>(eb + (col / 64) * C::kBlockBytes + comm_chunk_offset(r, (col % 64) / 8)) =
              make_uint4(e[0], e[1], e[2], e[3]);
        }
      }
      // decode weights of this row: 2^(s log2e - rowmax), normalised below
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < C::kCols; ++j) {
        x[j] = ptx::ex2(fmaf(x[j], kLog2e, -rowmax));
        sum += x[j];
      }
      xs[cq * 128 + r] = sum;
      asm volatile("bar.sync %0, 128;" ::"r"(bar_id) : "memory");
      const float inv = valid ? 1.f / ((xs[r] + xs[128 + r]) + (xs[256 + r] + xs[384 + r])) : 0.f;
      // the previous tile's MMA has read the P buffer
      if (t > 0 && !__all_sync(0xffffffffu, ptx::mbar_wait(P_free, (t - 1) & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      // P: chunks of 8 latents into the column blocks of 64
#pragma unroll
      for (int c = 0; c < C::kCols / 8; ++c) {
        const int col = c0 + 8 * c;  // first latent of the chunk
        uint4 v;
        v.x = ptx::pack_f16(x[8 * c + 0] * inv, x[8 * c + 1] * inv);
        v.y = ptx::pack_f16(x[8 * c + 2] * inv, x[8 * c + 3] * inv);
        v.z = ptx::pack_f16(x[8 * c + 4] * inv, x[8 * c + 5] * inv);
        v.w = ptx::pack_f16(x[8 * c + 6] * inv, x[8 * c + 7] * inv);
        *reinterpret_cast<uint4*>(smem + C::kOffP + (col / 64) * C::kBlockBytes + comm_chunk_offset(r, (col % 64) / 8)) =
            v;
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
