// FLARE decode on tcgen05 tensor cores.
//
// Y[n] = softmax_m(k_n . q_m) Z, one row per token, softmax over the M
// latents with scale 1.  "FLARE: Fast Low-rank Attention Routing Engine"
// review page, section "Основной механизм FLARE", decode step
// Y = SDPA(K, Q, Z, s=1); in FLARE++ the keys of the latents are the
// synthesised routing queries Q_dyn ("FLARE++: Low-rank attention with dynamic
// attention routing", "Méthodologie : FLARE++", routing encode-decode).
//
// Work of one CTA: one (b, h), Q and Z of that head resident in shared
// memory, and a contiguous run of 128-token tiles.
//   warp 0      TMA producer: Q and Z once, then K tiles into an NS-deep ring
//   warp 1      TMEM allocator + tcgen05.mma issuer of slot 0 (one thread)
//   warp 2      tcgen05.mma issuer of slot 1 (one thread)
//   warps 4-7   epilogue warpgroup of slot 0 (even tiles), one thread per token
//   warps 8-11  epilogue warpgroup of slot 1 (odd tiles)
// The slots own disjoint TMEM columns and each has its own issuer, so one
// slot's waits never hold up the other slot's MMAs.
// Per tile: S = K_tile Q^T (128 x MP, fp32, TMEM), the owning thread takes
// the max over its row's M valid latents, writes P = 2^(s log2e - max) as bf16
// over the first MP/2 columns, then O = P Z (128 x D) lands in columns
// [128, 128 + D) of the slot; the thread scales by 1/sum and stores its
// token's row of Y as bf16.
//
// TMEM: slot s owns columns [256 s, 256 s + 256).
#pragma once

#include "common.cuh"

namespace flare {

struct DecodeArgs {
  int N;
  int M;
  int q_batched;  // Q indexed by bh (1) or h = bh % H (0)
  int H;
  int splits;
  int tiles;
  __nv_bfloat16* Y;  // [BH][N][D]
  int* status;
  unsigned long long wait_ns;
};

template <int D, int MP, int NS>
struct DecodeCfg {
  using G = TileGeom<D>;
  static_assert(MP == 128 || MP == 256, "padded latent count");
  static constexpr int kLatBytes = G::bytes(MP);
  static constexpr int kTileBytes = G::bytes(kTileN);
  static constexpr int kOffQ = 0;
  static constexpr int kOffZ = kLatBytes;
  static constexpr int kOffStages = 2 * kLatBytes;
  static constexpr int kOffBars = kOffStages + NS * kTileBytes;
  // full[NS], empty[NS], qz_full, S_full[2], P_full[2], O_full[2], O_free[2], drain
  static constexpr int kNumBars = 2 * NS + 10;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSlotCols = 256;
  static constexpr uint32_t kColO = 128;  // O inside a slot
  static_assert(MP / 2 <= kColO && kColO + D <= kSlotCols, "TMEM slot layout");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16(kTileN, MP, 0, 0);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16(kTileN, D, 0, 1);
};

template <int D, int MP, int NS>
__global__ void __launch_bounds__(384, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmZ, const DecodeArgs args) {
  using C = DecodeCfg<D, MP, NS>;
  using G = typename C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* qz_full = bars + 2 * NS;
  uint64_t* S_full = bars + 2 * NS + 1;
  uint64_t* P_full = bars + 2 * NS + 3;
  uint64_t* O_full = bars + 2 * NS + 5;
  uint64_t* O_free = bars + 2 * NS + 7;
  uint64_t* drain = bars + 2 * NS + 9;
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
    ptx::mbar_init(qz_full, 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&S_full[s], 1);
      ptx::mbar_init(&P_full[s], 4);
      ptx::mbar_init(&O_full[s], 1);
      ptx::mbar_init(&O_free[s], 4);
    }
    ptx::mbar_init(drain, 2);  // one commit per issuer
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
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmQ);
      ptx::prefetch_tmap(&tmZ);
      const int qidx = args.q_batched ? bh : bh % args.H;
      ptx::mbar_arrive_expect_tx(qz_full, 2 * C::kLatBytes);
      for (int h = 0; h < MP / kLatRows; ++h)
        for (int b = 0; b < G::kBlocks; ++b) {
          const int off = b * MP * 128 + h * kLatRows * G::kRowBytes;
          ptx::tma_load_3d(smem + C::kOffQ + off, &tmQ, qz_full, b * 64, h * kLatRows, qidx);
          ptx::tma_load_3d(smem + C::kOffZ + off, &tmZ, qz_full, b * 64, h * kLatRows, bh);
        }
      const uint64_t pol = ptx::policy_evict_first();
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % NS;
        if (t >= NS && !ptx::mbar_wait(&empty[st], ((t / NS) - 1) & 1, s_abort, args.wait_ns)) {
          record_error(args.status, kErrTimeout, kSiteDecProducer);
          *s_abort = 1;
          break;
        }
        uint8_t* sk = smem + C::kOffStages + st * C::kTileBytes;
        ptx::mbar_arrive_expect_tx(&full[st], C::kTileBytes);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sk + b * kTileN * 128, &tmK, &full[st], b * 64, (tile0 + t) * kTileN, bh, pol);
        issued = t + 1;
      }
      ptx::mbar_wait_drain(qz_full, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        ptx::mbar_wait_drain(&full[t % NS], (t / NS) & 1);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------ MMA issuers (one per slot)
    if (lane == 0) {
      static_assert((NS & (NS - 1)) == 0, "ring depth must be a power of two");
      const int slot = warp - 1;
      bool ok = ptx::mbar_wait(qz_full, 0, s_abort, args.wait_ns);
      ptx::tc_fence_after();
      // descriptors of stage 0 / K step 0; stages and K steps only move the start address
      const uint64_t dK0 = G::kmajor(sbase + C::kOffStages, kTileN, 0);
      const uint64_t dQ0 = G::kmajor(sbase + C::kOffQ, MP, 0);
      const uint64_t dZ0 = G::mnmajor(sbase + C::kOffZ, MP, 0);
      const uint32_t tS = tmem + slot * C::kSlotCols;
      // The issuing thread stalls on any shared-memory access until its own
      // MMAs have completed: waits go before each group of MMAs.
      auto wait_stage = [&](int t) -> bool {
        return ptx::mbar_wait(&full[t & (NS - 1)], (t / NS) & 1, s_abort, args.wait_ns);
      };
      auto issue_qk = [&](int t) {
        const int st = t & (NS - 1);
        const uint64_t dK = dK0 + static_cast<uint32_t>(st * (C::kTileBytes >> 4));
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          ptx::mma_ss(tS, dK + G::kmajor_step(kTileN, k), dQ0 + G::kmajor_step(MP, k), C::kIdescQK, k > 0 ? 1u : 0u);
        ptx::mma_commit(&S_full[slot]);
        ptx::mma_commit(&empty[st]);
      };
      auto issue_pv = [&]() {
#pragma unroll
        for (int k = 0; k < MP / 16; ++k)
          ptx::mma_ts(tS + C::kColO, tS + k * 8, dZ0 + G::mnmajor_step(k), C::kIdescPV, k > 0 ? 1u : 0u);
        ptx::mma_commit(&O_full[slot]);
      };
      // this slot's tiles: t = slot + 2 i
      if (ok && slot < T) {
        ok = wait_stage(slot);
        if (ok) {
          ptx::tc_fence_after();
          issue_qk(slot);
        }
      }
      for (int i = 0; ok && slot + 2 * i < T; ++i) {
        const int t = slot + 2 * i;
        ok = (t + 2 >= T || wait_stage(t + 2)) && ptx::mbar_wait(&P_full[slot], i & 1, s_abort, args.wait_ns);
        if (!ok) break;
        ptx::tc_fence_after();
        issue_pv();
        if (t + 2 < T) {
          // the slot's columns are reused once its epilogue has read O of tile t
          ok = ptx::mbar_wait(&O_free[slot], i & 1, s_abort, args.wait_ns);
          if (ok) {
            ptx::tc_fence_after();
            issue_qk(t + 2);
          }
        }
      }
      if (!ok) {
        record_error(args.status, kErrTimeout, kSiteDecMma);
        *s_abort = 1;
      }
      ptx::mma_commit(drain);
      ptx::mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax / epilogue warpgroups
    const int s = (warp - 4) >> 2;
    const int r = (warp & 3) * 32 + lane;  // token row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + s * C::kSlotCols;
    const uint32_t tO = tS + C::kColO;
    const int count = s == 0 ? (T + 1) / 2 : T / 2;
    const int M = args.M;
    bool ok = true;
    for (int i = 0; i < count; ++i) {
      const int t = 2 * i + s;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&S_full[s], i & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // pass 1: row max over the M valid latents (columns >= M are padding;
      // M is a multiple of 16, so validity is uniform per 16-column group)
      float pm[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) pm[j] = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < MP; c0 += 128) {
        float x[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tmem_ld32(tS + c0 + 32 * c, x + 32 * c);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 8; ++g)
          if (c0 + 16 * g < M) {
#pragma unroll
            for (int j = 0; j < 8; ++j) pm[j] = ptx::max3(pm[j], x[16 * g + 2 * j], x[16 * g + 2 * j + 1]);
          }
      }
      const float mref =
          ptx::max3(ptx::max3(pm[0], pm[1], pm[2]), ptx::max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7])) * kLog2e;
      // pass 2: P = 2^(s log2e - mref) as bf16 pairs over the first MP/2 columns
      // (P of columns [c0, c0+64) lands in [c0/2, c0/2+32), already read)
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c0 = 0; c0 < MP; c0 += 64) {
        float x[64];
        ptx::tmem_ld32(tS + c0, x);
        ptx::tmem_ld32(tS + c0 + 32, x + 32);
        ptx::tmem_wait_ld();
        uint32_t p[32];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          if (c0 + 16 * g < M) {
#pragma unroll
            for (int c = 16 * g; c < 16 * g + 16; c += 2) {
              const float p0 = ptx::ex2(fmaf(x[c], kLog2e, -mref));
              const float p1 = ptx::ex2(fmaf(x[c + 1], kLog2e, -mref));
              ps[(c / 2) & 7] += p0 + p1;
              p[c / 2] = ptx::pack_bf16(p0, p1);
            }
          } else {
#pragma unroll
            for (int c = 16 * g; c < 16 * g + 16; c += 2) p[c / 2] = 0u;
          }
        }
        ptx::tmem_st32(tS + c0 / 2, p);
      }
      const float l = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&P_full[s]);

      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&O_full[s], i & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float o[D];
      if constexpr (D >= 32) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) ptx::tmem_ld32(tO + 32 * c, o + 32 * c);
      } else {
        ptx::tmem_ld16(tO, o);
      }
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&O_free[s]);

      const long long tok = static_cast<long long>(tile0 + t) * kTileN + r;
      if (tok < args.N) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(args.Y + (static_cast<size_t>(bh) * args.N + tok) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint4 v;
          v.x = ptx::pack_bf16(o[8 * c + 0] * inv, o[8 * c + 1] * inv);
          v.y = ptx::pack_bf16(o[8 * c + 2] * inv, o[8 * c + 3] * inv);
          v.z = ptx::pack_bf16(o[8 * c + 4] * inv, o[8 * c + 5] * inv);
          v.w = ptx::pack_bf16(o[8 * c + 6] * inv, o[8 * c + 7] * inv);
          dst[c] = v;
        }
      }
    }
    if (!ok) {
      record_error(args.status, kErrTimeout, kSiteDecSoftmax);
      *s_abort = 1;
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
