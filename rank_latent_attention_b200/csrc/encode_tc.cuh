// FLARE encode on tcgen05 tensor cores, split over the token axis.
//
// Computes, per head (b, h) and per split of the N tokens, the unnormalised
// softmax partials of Z = softmax(Q K^T) V with the softmax over tokens:
//   O_part[m][:] = sum_n 2^(s_mn log2e - mref_m) V[n][:],
//   l_part[m]    = sum_n 2^(s_mn log2e - mref_m),   m_part[m] = mref_m,
// where s_mn = q_m . k_n (scale 1).  "FLARE: Fast Low-rank Attention Routing
// Engine" review page, section "Основной механизм FLARE", encode step; the
// split-and-merge of softmax statistics is the exact reduction the FLARE++
// page ("Contributions Clés", context parallelism) exchanges between devices,
// applied here between CTAs of one GPU.  lse_merge (merge.cuh) combines the
// partials into the normalised M x D result.
//
// Work of one CTA: one (b, h) and a contiguous run of 128-token tiles.
//   warp 0      TMA producer: Q halves once, then K/V tiles into an NS-deep ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 4-7   softmax warpgroup of slot 0 (one thread per latent row)
//   warps 8-11  softmax warpgroup of slot 1
// With M > 128 the two slots are the two 128-row halves of the latents and
// both see every tile; with M <= 128 both slots use the same latents and take
// alternate tiles, each keeping its own partial.  While one warpgroup turns
// its S tile into P, the tensor core runs the other slot's GEMMs.
//
// TMEM columns: S of slot s at [128 s, 128 s + 128) (fp32); P (bf16 pairs)
// overwrites the first 64 columns of its S after the scores are read; O of
// slot s at [256 + D s, 256 + D s + D).
//
// Online softmax with a lazy reference: a row's reference max only moves
// when a tile's max exceeds it by more than 2^8, so the O rescale in tensor
// memory is rare.  Any reference gives the same normalised result because
// P and l use the same one.
#pragma once

#include "common.cuh"

namespace flare {

struct EncodeArgs {
  int N;          // tokens per head
  int M;          // latents
  int q_batched;  // Q indexed by bh (1) or by h = bh % H (0)
  int H;
  int splits;     // CTAs per head (gridDim.x)
  int tiles;      // ceil(N / 128)
  int P;          // partials per head
  float* O_part;  // [BH][P][M][D]
  float* m_part;  // [BH][P][M]  (log2 domain)
  float* l_part;  // [BH][P][M]
  int* status;    // device status word {code, site}
  unsigned long long wait_ns;
};

template <int D, int NHALF, int NS>
struct EncodeCfg {
  using G = TileGeom<D>;
  static constexpr int kThreads = 384;
  static constexpr int kQHalfBytes = G::bytes(kLatRows);
  static constexpr int kTileBytes = G::bytes(kTileN);
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffStages = kOffQ + NHALF * kQHalfBytes;
  static constexpr int kOffBars = kOffStages + NS * kStageBytes;
  // full[NS], empty[NS], q_full, S_full[2], P_full[2], O_final[2], drain
  static constexpr int kNumBars = 2 * NS + 8;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-B alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = kTileN, kColO0 = 2 * kTileN, kColO1 = 2 * kTileN + D;
  static_assert(2 * kTileN + 2 * D <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16(kLatRows, kTileN, 0, 0);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16(kLatRows, D, 0, 1);
};

template <int D, int NHALF, int NS>
__global__ void __launch_bounds__(384, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const EncodeArgs args) {
  using C = EncodeCfg<D, NHALF, NS>;
  using G = typename C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_full = bars + 2 * NS;
  uint64_t* S_full = bars + 2 * NS + 1;
  uint64_t* P_full = bars + 2 * NS + 3;
  uint64_t* O_final = bars + 2 * NS + 5;
  uint64_t* drain = bars + 2 * NS + 7;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int tile0 = static_cast<int>((static_cast<long long>(split) * args.tiles) / args.splits);
  const int tile1 = static_cast<int>((static_cast<long long>(split + 1) * args.tiles) / args.splits);
  const int T = tile1 - tile0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], 1);
    }
    ptx::mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&S_full[s], 1);
      ptx::mbar_init(&P_full[s], 4);  // one arrival per softmax warp
      ptx::mbar_init(&O_final[s], 1);
    }
    ptx::mbar_init(drain, 1);
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(s_tmem, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = ptx::smem_u32(smem);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmQ);
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmV);
      const int qidx = args.q_batched ? bh : bh % args.H;
      ptx::mbar_arrive_expect_tx(q_full, NHALF * C::kQHalfBytes);
      for (int h = 0; h < NHALF; ++h)
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d(smem + C::kOffQ + h * C::kQHalfBytes + b * kLatRows * 128, &tmQ, q_full, b * 64,
                           h * kLatRows, qidx);
      const uint64_t pol = ptx::policy_evict_first();
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % NS;
        if (t >= NS && !ptx::mbar_wait(&empty[st], ((t / NS) - 1) & 1, s_abort, args.wait_ns)) {
          record_error(args.status, kErrTimeout, kSiteEncProducer);
          *s_abort = 1;
          break;
        }
        uint8_t* sk = smem + C::kOffStages + st * C::kStageBytes;
        uint8_t* sv = sk + C::kTileBytes;
        const int tok = (tile0 + t) * kTileN;
        ptx::mbar_arrive_expect_tx(&full[st], C::kStageBytes);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sk + b * kTileN * 128, &tmK, &full[st], b * 64, tok, bh, pol);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sv + b * kTileN * 128, &tmV, &full[st], b * 64, tok, bh, pol);
        issued = t + 1;
      }
      // Every load issued must land before the CTA may exit (matters on the abort path only).
      ptx::mbar_wait_drain(q_full, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        ptx::mbar_wait_drain(&full[t % NS], (t / NS) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = ptx::mbar_wait(q_full, 0, s_abort, args.wait_ns);
      ptx::tc_fence_after();
      const uint32_t sQ = sbase + C::kOffQ;
      auto stage_k = [&](int t) { return sbase + C::kOffStages + (t % NS) * C::kStageBytes; };
      const uint32_t colS[2] = {C::kColS0, C::kColS1};
      const uint32_t colO[2] = {C::kColO0, C::kColO1};

      auto issue_qk = [&](int t, int s) -> bool {
        if (!ptx::mbar_wait(&full[t % NS], (t / NS) & 1, s_abort, args.wait_ns)) return false;
        ptx::tc_fence_after();
        const uint32_t qh = sQ + (NHALF == 2 ? s : 0) * C::kQHalfBytes;
        const uint32_t kb = stage_k(t);
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          ptx::mma_ss(tmem + colS[s], G::kmajor(qh, kLatRows, k), G::kmajor(kb, kTileN, k), C::kIdescQK,
                      k > 0 ? 1u : 0u);
        ptx::mma_commit(&S_full[s]);
        return true;
      };
      auto issue_pv = [&](int t, int s, int local) -> bool {
        if (!ptx::mbar_wait(&P_full[s], local & 1, s_abort, args.wait_ns)) return false;
        ptx::tc_fence_after();
        const uint32_t vb = stage_k(t) + C::kTileBytes;
#pragma unroll
        for (int k = 0; k < kTileN / 16; ++k)
          ptx::mma_ts(tmem + colO[s], tmem + colS[s] + k * 8, G::mnmajor(vb, kTileN, k), C::kIdescPV,
                      (local > 0 || k > 0) ? 1u : 0u);
        return true;
      };

      if (ok) {
        if (NHALF == 2) {
          ok = issue_qk(0, 0) && issue_qk(0, 1);
          for (int t = 0; ok && t < T; ++t) {
            for (int s = 0; ok && s < 2; ++s) {
              ok = issue_pv(t, s, t);
              if (!ok) break;
              if (s == 1) ptx::mma_commit(&empty[t % NS]);
              if (t + 1 < T)
                ok = issue_qk(t + 1, s);
              else
                ptx::mma_commit(&O_final[s]);
            }
          }
        } else {
          ok = issue_qk(0, 0) && (T < 2 || issue_qk(1, 1));
          for (int t = 0; ok && t < T; ++t) {
            const int s = t & 1;
            ok = issue_pv(t, s, t >> 1);
            if (!ok) break;
            ptx::mma_commit(&empty[t % NS]);
            if (t + 2 < T)
              ok = issue_qk(t + 2, s);
            else
              ptx::mma_commit(&O_final[s]);
          }
        }
      }
      if (!ok) {
        record_error(args.status, kErrTimeout, kSiteEncMma);
        *s_abort = 1;
      }
      // Drain: wait for every MMA issued by this thread before TMEM is released.
      ptx::mma_commit(drain);
      ptx::mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warpgroups
    const int s = (warp - 4) >> 2;     // slot
    const int r = (warp & 3) * 32 + lane;  // TMEM lane = latent row within the half
    const int m = (NHALF == 2 ? s * kLatRows : 0) + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + (s == 0 ? C::kColS0 : C::kColS1);
    const uint32_t tO = tmem + lane_off + (s == 0 ? C::kColO0 : C::kColO1);
    const int count = NHALF == 2 ? T : (s == 0 ? (T + 1) / 2 : T / 2);

    float mref = -INFINITY;  // reference max, log2 domain
    float l = 0.f;
    bool ok = true;
    for (int i = 0; i < count; ++i) {
      const int t = NHALF == 2 ? i : 2 * i + s;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&S_full[s], i & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float x[kTileN];
#pragma unroll
      for (int c = 0; c < kTileN / 32; ++c) ptx::tmem_ld32(tS + c * 32, x + c * 32);
      ptx::tmem_wait_ld();
      const int valid = args.N - (tile0 + t) * kTileN;
      if (valid < kTileN) {
#pragma unroll
        for (int c = 0; c < kTileN; ++c)
          if (c >= valid) x[c] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int c = 1; c < kTileN; ++c) mx = fmaxf(mx, x[c]);
      mx *= kLog2e;
      const bool need = mx > mref + 8.f;
      const float nref = need ? mx : mref;
      const float alpha = ptx::ex2(mref - nref);  // 0 on the first tile
      l *= alpha;
      mref = nref;
      {
        uint32_t p[kTileN / 2];
#pragma unroll
        for (int c = 0; c < kTileN; c += 2) {
          const float p0 = ptx::ex2(fmaf(x[c], kLog2e, -mref));
          const float p1 = ptx::ex2(fmaf(x[c + 1], kLog2e, -mref));
          l += p0 + p1;
          p[c / 2] = ptx::pack_bf16(p0, p1);
        }
#pragma unroll
        for (int c = 0; c < kTileN / 64; ++c) ptx::tmem_st32(tS + c * 32, p + c * 32);
      }
      // Rare: the reference moved, so rescale this row of O (no MMA touches
      // O now: the previous P.V completed before this tile's S was signalled,
      // and the next one waits for P_full).
      if (i > 0 && __any_sync(0xffffffffu, need)) {
        constexpr int kChunk = D < 32 ? D : 32;
#pragma unroll
        for (int c = 0; c < D / kChunk; ++c) {
          float o[kChunk];
          if constexpr (kChunk == 32) ptx::tmem_ld32(tO + c * 32, o); else ptx::tmem_ld16(tO, o);
          ptx::tmem_wait_ld();
          uint32_t u[kChunk];
#pragma unroll
          for (int j = 0; j < kChunk; ++j) u[j] = __float_as_uint(o[j] * alpha);
          if constexpr (kChunk == 32) ptx::tmem_st32(tO + c * 32, u); else ptx::tmem_st16(tO, u);
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&P_full[s]);
    }

    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] = 0.f;
    if (ok && count > 0) {
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(&O_final[s], 0, s_abort, args.wait_ns));
      if (ok) {
        ptx::tc_fence_after();
        if constexpr (D >= 32) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) ptx::tmem_ld32(tO + c * 32, o + c * 32);
        } else {
          ptx::tmem_ld16(tO, o);
        }
        ptx::tmem_wait_ld();
      }
    }
    if (!ok) {
      record_error(args.status, kErrTimeout, kSiteEncSoftmax);
      *s_abort = 1;
    } else if (m < args.M) {
      const int p = NHALF == 2 ? split : 2 * split + s;
      const size_t row = (static_cast<size_t>(bh) * args.P + p) * args.M + m;
      float4* dst = reinterpret_cast<float4*>(args.O_part + row * D);
#pragma unroll
      for (int c = 0; c < D / 4; ++c) dst[c] = make_float4(o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
      args.m_part[row] = count > 0 ? mref : -INFINITY;
      args.l_part[row] = l;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace flare
