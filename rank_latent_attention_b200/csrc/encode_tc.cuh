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
// applied here between CTAs of one GPU (and between the accumulators of one
// CTA).  lse_merge (merge.cuh) combines the partials into the normalised
// M x D result.
//
// Work of one CTA: one (b, h) and a contiguous run of 64-token tiles.
//   warp 0            TMA producer: Q once, then K/V tiles into an NS-deep ring
//   warps 1-3, 12     tcgen05.mma issuers, one thread each (warp 1 also
//                     allocates TMEM)
//   warps 4-7         softmax warpgroup of slot 0 (one thread per latent row)
//   warps 8-11        softmax warpgroup of slot 1
// With M > 128 the two slots are the two 128-row halves of the latents and
// both see every tile; with M <= 128 both slots use the same latents and take
// alternate tiles.
//
// Each slot has NB buffers (2 for D <= 64, 1 for D = 128) taken round robin by
// its tiles, and each (slot, buffer) pair owns an S region, an O accumulator,
// its own online-softmax state and its own issuer thread.  An issuer waits for
// P of its buffer, issues P.V into its O and Q.K^T of the buffer's next tile,
// and commits.  Why one issuer per buffer: a thread that has MMAs in flight
// stalls on any synchronising instruction until they complete, so a thread
// serving several buffers would couple their latencies; with one per buffer
// the path P(t) -> P.V(t) -> Q.K^T(t + NB) -> S ready has the other buffer's
// tile of softmax time to complete in.  S of a buffer's tile being ready also
// means the buffer's previous P.V is done (one thread, in order), which is
// all the rare O rescale needs.
//
// TMEM columns: S of (slot s, buffer b) at [64 (NB s + b), +64) fp32; P (bf16
// pairs) overwrites the first 32 columns of its S after the scores are read;
// O of (s, b) at [128 NB + D (NB s + b), +D).  Q stays in shared memory.
//
// Online softmax with a lazy reference: a row's reference max only moves when
// a tile's max exceeds it by more than 2^8, so the O rescale in tensor memory
// is rare.  Any reference gives the same normalised result because P and l
// use the same one.
#pragma once

#include "common.cuh"

namespace flare {

constexpr int kEncTile = 64;  // tokens per encode tile

struct EncodeArgs {
  int N;          // tokens per head
  int M;          // latents
  int q_batched;  // Q indexed by bh (1) or by h = bh % H (0)
  int H;
  int splits;     // CTAs per head (gridDim.x)
  int tiles;      // ceil(N / 64)
  int P;          // partials per head
  float* O_part;  // [BH][P][M][D]
  float* m_part;  // [BH][P][M]  (log2 domain)
  float* l_part;  // [BH][P][M]
  int* status;    // device status word {code, site}
  unsigned long long wait_ns;
};

// Buffers (and accumulators) per slot of the encode for head dim D.
__host__ __device__ constexpr int encode_buffers(int D) { return D <= 64 ? 2 : 1; }

// Partials per (head, split) written by encode_tc_kernel.
__host__ __device__ constexpr int encode_partials_per_split(int D, int nhalf) {
  return encode_buffers(D) * (nhalf == 2 ? 1 : 2);
}

template <int D, int NHALF, int NS>
struct EncodeCfg {
  using G = TileGeom<D>;
  static constexpr int NB = encode_buffers(D);
  static constexpr int kThreads = 416;
  static constexpr int kQHalfBytes = G::bytes(kLatRows);
  static constexpr int kTileBytes = G::bytes(kEncTile);
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kOffQ = 0;
  static constexpr int kOffStages = NHALF * kQHalfBytes;
  static constexpr int kOffBars = kOffStages + NS * kStageBytes;
  // full[NS], empty[NS], q_ready, S_full[2 NB], P_full[2 NB], O_final[2 NB], drain
  static constexpr int kNumBars = 2 * NS + 2 + 6 * NB;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-B alignment
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 2 * NB * kEncTile;
  static_assert(kColO + 2 * NB * D <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static_assert((NS & (NS - 1)) == 0, "ring depth must be a power of two");
  // An issuer at tile t waits for its buffer's next tile, NB (M > 128) or 2 NB
  // (M <= 128) tiles ahead, whose stage is free once tile t - 1 is released.
  static_assert(NS >= (NHALF == 2 ? NB : 2 * NB) + 1, "ring too shallow for the look-ahead");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16(kLatRows, kEncTile, 0, 0);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16(kLatRows, D, 0, 1);
  __host__ __device__ static constexpr uint32_t col_s(int slot, int buf) { return (NB * slot + buf) * kEncTile; }
  __host__ __device__ static constexpr uint32_t col_o(int slot, int buf) { return kColO + (NB * slot + buf) * D; }
};

template <int D, int NHALF, int NS>
__global__ void __launch_bounds__(416, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const EncodeArgs args) {
  using C = EncodeCfg<D, NHALF, NS>;
  using G = typename C::G;
  constexpr int NB = C::NB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_ready = bars + 2 * NS;
  uint64_t* S_full = bars + 2 * NS + 1;            // [NB slot + buf]
  uint64_t* P_full = bars + 2 * NS + 1 + 2 * NB;   // [NB slot + buf]
  uint64_t* O_final = bars + 2 * NS + 1 + 4 * NB;  // [NB slot + buf]
  uint64_t* drain = bars + 2 * NS + 1 + 6 * NB;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int tile0 = static_cast<int>((static_cast<long long>(split) * args.tiles) / args.splits);
  const int tile1 = static_cast<int>((static_cast<long long>(split + 1) * args.tiles) / args.splits);
  const int T = tile1 - tile0;
  // tiles of slot s (its local tile i is tile NHALF == 2 ? i : s + 2 i)
  auto count_of = [&](int s) { return NHALF == 2 ? T : (s == 0 ? (T + 1) / 2 : T / 2); };
  auto tile_of = [&](int s, int i) { return NHALF == 2 ? i : s + 2 * i; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      ptx::mbar_init(&full[i], 1);
      ptx::mbar_init(&empty[i], NHALF == 2 ? 2 : 1);  // both slots read every stage when M > 128
    }
    ptx::mbar_init(q_ready, 1);
    for (int i = 0; i < 2 * NB; ++i) {
      ptx::mbar_init(&S_full[i], 1);
      ptx::mbar_init(&P_full[i], 4);  // one arrival per softmax warp of the slot
      ptx::mbar_init(&O_final[i], 1);
    }
    ptx::mbar_init(drain, 2 * NB);  // one commit per issuer
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
  // issuer index of this warp (-1: not an issuer)
  const int issuer = warp == 1 ? 0 : warp == 2 ? 1 : warp == 3 ? 2 : warp == 12 ? 3 : -1;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const int qidx = args.q_batched ? bh : bh % args.H;
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmV);
      ptx::prefetch_tmap(&tmQ);
      ptx::mbar_arrive_expect_tx(q_ready, NHALF * C::kQHalfBytes);
      for (int h = 0; h < NHALF; ++h)
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d(smem + C::kOffQ + h * C::kQHalfBytes + b * kLatRows * 128, &tmQ, q_ready, b * 64,
                           h * kLatRows, qidx);
      const uint64_t pol = ptx::policy_evict_first();
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t & (NS - 1);
        if (t >= NS && !ptx::mbar_wait(&empty[st], ((t / NS) - 1) & 1, s_abort, args.wait_ns)) {
          record_error(args.status, kErrTimeout, kSiteEncProducer);
          *s_abort = 1;
          break;
        }
        uint8_t* sk = smem + C::kOffStages + st * C::kStageBytes;
        uint8_t* sv = sk + C::kTileBytes;
        const int tok = (tile0 + t) * kEncTile;
        ptx::mbar_arrive_expect_tx(&full[st], C::kStageBytes);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sk + b * kEncTile * 128, &tmK, &full[st], b * 64, tok, bh, pol);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sv + b * kEncTile * 128, &tmV, &full[st], b * 64, tok, bh, pol);
        issued = t + 1;
      }
      // Every load issued must land before the CTA may exit (matters on the abort path only).
      ptx::mbar_wait_drain(q_ready, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        ptx::mbar_wait_drain(&full[t & (NS - 1)], (t / NS) & 1);
    }
  } else if (issuer >= 0) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0 && issuer < 2 * NB) {
      const int s = issuer / NB;  // slot
      const int b = issuer % NB;  // buffer
      const int count = count_of(s);
      const int half = NHALF == 2 ? s : 0;
      bool ok = true;
      if (b < count) {
        // Descriptors of stage 0 / K step 0; a stage adds kStageBytes >> 4 to
        // the start-address field, a K step adds a compile-time constant.
        const uint64_t dK0 = G::kmajor(sbase + C::kOffStages, kEncTile, 0);
        const uint64_t dV0 = G::mnmajor(sbase + C::kOffStages + C::kTileBytes, kEncTile, 0);
        const uint64_t dQ = G::kmajor(sbase + C::kOffQ + half * C::kQHalfBytes, kLatRows, 0);
        const uint32_t tS = tmem + C::col_s(s, b);
        const uint32_t tO = tmem + C::col_o(s, b);
        auto wait_stage = [&](int t) -> bool {
          return ptx::mbar_wait(&full[t & (NS - 1)], (t / NS) & 1, s_abort, args.wait_ns);
        };
        auto issue_qk = [&](int t) {
          const uint64_t dK = dK0 + static_cast<uint32_t>((t & (NS - 1)) * (C::kStageBytes >> 4));
#pragma unroll
          for (int k = 0; k < D / 16; ++k)
            ptx::mma_ss(tS, dQ + G::kmajor_step(kLatRows, k), dK + G::kmajor_step(kEncTile, k), C::kIdescQK,
                        k > 0 ? 1u : 0u);
          ptx::mma_commit(&S_full[issuer]);
        };
        ok = ptx::mbar_wait(q_ready, 0, s_abort, args.wait_ns) && wait_stage(tile_of(s, b));
        if (ok) {
          ptx::tc_fence_after();
          issue_qk(tile_of(s, b));
        }
        // this buffer's tiles: local i = b + NB k
        for (int i = b, k = 0; ok && i < count; i += NB, ++k) {
          const int t = tile_of(s, i);
          const int tn = i + NB < count ? tile_of(s, i + NB) : -1;
          // every wait before the MMAs: a wait after them would stall until they complete
          ok = (tn < 0 || wait_stage(tn)) && ptx::mbar_wait(&P_full[issuer], k & 1, s_abort, args.wait_ns);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint64_t dV = dV0 + static_cast<uint32_t>((t & (NS - 1)) * (C::kStageBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < kEncTile / 16; ++kk)
            ptx::mma_ts(tO, tS + kk * 8, dV + G::mnmajor_step(kk), C::kIdescPV, (k > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_commit(&empty[t & (NS - 1)]);
          if (tn >= 0)
            issue_qk(tn);  // reuses S of tile t: after its P.V in issue order
          else
            ptx::mma_commit(&O_final[issuer]);
        }
      }
      if (!ok) {
        record_error(args.status, kErrTimeout, kSiteEncMma);
        *s_abort = 1;
      }
      // Drain: wait for every MMA issued by the issuers before TMEM is released.
      ptx::mma_commit(drain);
      ptx::mbar_wait_drain(drain, 0);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ softmax warpgroups
    const int s = (warp - 4) >> 2;         // slot
    const int r = (warp & 3) * 32 + lane;  // TMEM lane = latent row within the half
    const int m = (NHALF == 2 ? s : 0) * kLatRows + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int count = count_of(s);

    float mref[NB], l[NB];  // per-buffer reference max (log2 domain) and running sum
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      mref[b] = -INFINITY;
      l[b] = 0.f;
    }
    bool ok = true;
    for (int i0 = 0; ok && i0 < count; i0 += NB) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const int i = i0 + b;
        if (i >= count) break;
        const int k = i0 / NB;  // index of the tile among the buffer's tiles
        const int t = tile_of(s, i);
        const int q = NB * s + b;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait(&S_full[q], k & 1, s_abort, args.wait_ns))) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tS = tmem + lane_off + C::col_s(s, b);
        float x[kEncTile];
        ptx::tmem_ld32(tS, x);
        ptx::tmem_ld32(tS + 32, x + 32);
        ptx::tmem_wait_ld();
        const int valid = args.N - (tile0 + t) * kEncTile;
        if (valid < kEncTile) {
#pragma unroll
          for (int c = 0; c < kEncTile; ++c)
            if (c >= valid) x[c] = -INFINITY;
        }
        // row max as 8 independent 3-input chains
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = fmaxf(x[2 * u], x[2 * u + 1]);
#pragma unroll
        for (int c = 16; c < kEncTile; c += 16)
#pragma unroll
          for (int u = 0; u < 8; ++u) pm[u] = ptx::max3(pm[u], x[c + 2 * u], x[c + 2 * u + 1]);
        const float mx =
            ptx::max3(ptx::max3(pm[0], pm[1], pm[2]), ptx::max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7])) * kLog2e;
        const bool need = mx > mref[b] + 8.f;
        const float nref = need ? mx : mref[b];
        const float alpha = ptx::ex2(mref[b] - nref);  // 0 on the buffer's first tile
        l[b] *= alpha;
        mref[b] = nref;
        {
          uint32_t p[kEncTile / 2];
          float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // independent partial sums
#pragma unroll
          for (int c = 0; c < kEncTile; c += 2) {
            const float p0 = ptx::ex2(fmaf(x[c], kLog2e, -nref));
            const float p1 = ptx::ex2(fmaf(x[c + 1], kLog2e, -nref));
            ps[(c / 2) & 7] += p0 + p1;
            p[c / 2] = ptx::pack_bf16(p0, p1);
          }
          ptx::tmem_st32(tS, p);
          l[b] += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        }
        // Rare: the reference moved, so rescale this row of the buffer's O.
        // No MMA writes it now: its previous P.V completed before this S was
        // signalled (same issuer, in order) and its next one waits for P_full.
        if (k > 0 && __any_sync(0xffffffffu, need)) {
          const uint32_t tO = tmem + lane_off + C::col_o(s, b);
          constexpr int kChunk = D < 32 ? D : 32;
#pragma unroll
          for (int c = 0; c < D / kChunk; ++c) {
            float o[kChunk];
            if constexpr (kChunk == 32) ptx::tmem_ld32(tO + c * 32, o); else ptx::tmem_ld16(tO, o);
            ptx::tmem_wait_ld();
            uint32_t u[kChunk];
#pragma unroll
            for (int z = 0; z < kChunk; ++z) u[z] = __float_as_uint(o[z] * alpha);
            if constexpr (kChunk == 32) ptx::tmem_st32(tO + c * 32, u); else ptx::tmem_st16(tO, u);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&P_full[q]);
      }
    }

    // Epilogue: one partial per (slot, buffer); O streamed out of TMEM in chunks.
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const bool has = b < count;
      if (ok && has) {
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&O_final[NB * s + b], 0, s_abort, args.wait_ns));
        if (ok) ptx::tc_fence_after();
      }
      if (!ok) break;
      const int p = NHALF == 2 ? split * NB + b : (split * 2 + s) * NB + b;
      const size_t row = (static_cast<size_t>(bh) * args.P + p) * args.M + m;
      float4* dst = reinterpret_cast<float4*>(args.O_part + row * D);
      const uint32_t tO = tmem + lane_off + C::col_o(s, b);
      constexpr int kChunk = D < 32 ? D : 32;
#pragma unroll
      for (int c = 0; c < D / kChunk; ++c) {
        float o[kChunk];
        if (has) {
          if constexpr (kChunk == 32) ptx::tmem_ld32(tO + c * 32, o); else ptx::tmem_ld16(tO, o);
          ptx::tmem_wait_ld();
        } else {
#pragma unroll
          for (int z = 0; z < kChunk; ++z) o[z] = 0.f;
        }
        if (m < args.M) {
#pragma unroll
          for (int z = 0; z < kChunk / 4; ++z)
            dst[c * (kChunk / 4) + z] = make_float4(o[4 * z], o[4 * z + 1], o[4 * z + 2], o[4 * z + 3]);
        }
      }
      if (m < args.M) {
        args.m_part[row] = has ? mref[b] : -INFINITY;
        args.l_part[row] = has ? l[b] : 0.f;
      }
    }
    if (!ok) {
      record_error(args.status, kErrTimeout, kSiteEncSoftmax);
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
