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
// Work of one CTA: one (b, h) and a contiguous run of 64-token tiles.
//   warps 0-15   four softmax warpgroups (slot s, column half c): thread r of
//                group (s, c) owns latent row r of slot s and columns
//                [32 c, 32 c + 32) of every tile of the slot
//   warp 16      TMA producer: K/V tiles into an NS-deep ring (and Q when it
//                stays in shared memory); also allocates TMEM
//   warps 17-18  tcgen05.mma issuers, one warp per slot
// With M > 128 the two slots are the two 128-row halves of the latents and
// both see every tile; with M <= 128 both slots use the same latents and take
// alternate tiles.
//
// Per slot, S is double-buffered in TMEM: while the two groups turn S(i) into
// P(i), the MMAs of tile i + 1 are already done, and the issuer, once P(i) is
// stored, issues P(i).V and Q.K^T of tile i + 2 into the freed buffer.  A
// thread with MMAs in flight stalls on its next synchronising instruction
// until they complete, which is why the issuers are warps of their own: their
// next wait (P of the following tile) is a whole softmax phase away.  An
// issuer warp runs its loop as a whole and issues under elect.sync, which
// keeps the MMA operands warp-uniform (issue from one divergent thread runs
// well below the tensor pipe's rate).  Slot 1 starts half a phase late so
// the two slots' softmax phases interleave.
//
// D <= 64: each group has its own O accumulator and reference max, so the
// groups never exchange data within a tile; the K steps of P.V over tokens
// [32 c, +32) go to accumulator (s, c), and the epilogue folds the two
// accumulators of a slot like any two partials.  D = 128 (TMEM too small for
// four accumulators): the two groups of a slot share O and agree on each
// row's reference through shared memory (a named barrier per tile).
//
// TMEM columns: S of (slot s, buffer j) at [64 (2 s + j), +64) fp32; group c
// writes its P (bf16 pairs) over [32 c, +16) of it, inside its own scores.
// O at [256 + D a, +D) for accumulator a = 2 s + c (D <= 64) or a = s
// (D = 128); Q after the accumulators as bf16 pairs when it fits (Q.K^T then
// reads it as the TMEM A operand), else in shared memory.
//
// Online softmax with a lazy reference.  Any reference gives the same
// normalised result because P and l use the same one, so a row's reference
// only has to keep 2^(x log2e - reference) inside the fp32 range:
//   - past the first tile (split accumulators), a group takes the exponentials
//     of a full tile against the reference it has, without the half-row max,
//     and keeps them if every row's sum stays within 2^32;
//   - otherwise (first tile, ragged tile, a sum above 2^32 or inf, or a shared
//     O) it takes the half-row max, and the reference moves to it when the max
//     exceeds the reference by more than 2^8; the O rescale in tensor memory
//     is rare.
// Of every 16 column pairs, those in kEncPolyPairs take their exponentials
// from exp2_poly3 (FMA pipe) instead of MUFU.
//
// Epilogue: each CTA writes one partial per head (O_part[split] etc.), the
// accumulators that cover the same latent rows folded with their weights
// 2^(mref_a - max_a mref_a).
//
// Split precision (PREC > 0, D <= 64).  bf16 operands carry 8 significant
// bits; for outputs whose largest values sit tens of times above their RMS
// that rounding alone exceeds a 2e-2 x RMS budget.  Each rounded operand x is
// then carried as the pair hi = bf16(x), lo = bf16(x - hi), which holds x to
// about 2^-17, and a product takes one MMA per pair member:
//   PREC >= 1: P = P_hi + P_lo, and O += P_hi V + P_lo V (V is an exact
//              bf16 input); P_hi over the first 16 of the group's 32 score
//              columns, P_lo over the other 16;
//   PREC == 2: the queries too (the routing encode's Q_dyn, given as a hi
//              and a lo array): S = Q_hi K^T + Q_lo K^T.
// Every exponential of a split-precision tile is taken on MUFU (the FMA-pipe
// polynomial's 7.5e-5 relative error would be the largest term left).
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace flare {

constexpr int kEncTile = 64;  // tokens per encode tile

struct EncodeArgs {
  const void* Q;  // bf16 [BH or H][M][D]: read into TMEM directly when D <= 64
  const void* Q_lo;  // split precision (PREC == 2): the low parts of Q, same layout
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
  // One split per head (splits == 1, P == 1): the CTA writes the normalised
  // result and the log-sum-exp itself, with the merge's own operations on
  // the same fp32 values (out = O / l, lse = (mref + log2 l) ln 2), instead
  // of a partial for lse_merge_kernel.
  int direct;
  void* out;                // [BH][M][D]: bf16, or fp32 when out_f32
  int out_f32;
  float* lse_out;           // [BH][M] natural log, or null
  __nv_bfloat16* out_hi;    // fp32 out only: the result as a bf16 pair hi + lo, or null
  __nv_bfloat16* out_lo;
};

// Stores n consecutive elements of one row of a direct encode's result:
// v = acc / l (0 when the row saw no token), as the merge forms it.
template <int n>
__device__ __forceinline__ void encode_store_direct(const EncodeArgs& a, size_t e0, const float* acc, float l) {
  float v[n];
#pragma unroll
  for (int z = 0; z < n; ++z) v[z] = l > 0.f ? acc[z] / l : 0.f;
  if (a.out_f32) {
    float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + e0);
#pragma unroll
    for (int z = 0; z < n / 4; ++z) o[z] = make_float4(v[4 * z], v[4 * z + 1], v[4 * z + 2], v[4 * z + 3]);
    if (a.out_hi) {
      uint32_t hi[n / 2], lo[n / 2];
#pragma unroll
      for (int z = 0; z < n / 2; ++z) {
        hi[z] = ptx::pack_bf16(v[2 * z], v[2 * z + 1]);
        lo[z] = ptx::pack_bf16(v[2 * z] - __uint_as_float(hi[z] << 16), v[2 * z + 1] - __uint_as_float(hi[z] & 0xffff0000u));
      }
      uint4* oh = reinterpret_cast<uint4*>(a.out_hi + e0);
      uint4* ol = reinterpret_cast<uint4*>(a.out_lo + e0);
#pragma unroll
      for (int z = 0; z < n / 8; ++z) {
        oh[z] = make_uint4(hi[4 * z], hi[4 * z + 1], hi[4 * z + 2], hi[4 * z + 3]);
        ol[z] = make_uint4(lo[4 * z], lo[4 * z + 1], lo[4 * z + 2], lo[4 * z + 3]);
      }
    }
  } else {
    uint32_t b[n / 2];
#pragma unroll
    for (int z = 0; z < n / 2; ++z) b[z] = ptx::pack_bf16(v[2 * z], v[2 * z + 1]);
    uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + e0);
#pragma unroll
    for (int z = 0; z < n / 8; ++z) o[z] = make_uint4(b[4 * z], b[4 * z + 1], b[4 * z + 2], b[4 * z + 3]);
  }
}

// Partials per (head, split) written by encode_tc_kernel.
__host__ __device__ constexpr int encode_partials_per_split(int /*D*/, int /*nhalf*/) { return 1; }

// Column pairs (bit j: pair j of each 16) whose exponentials go to
// exp2_poly3 instead of MUFU: pair 0, 1/16 of the tile.  Measured A/B on the
// million-token workload (same GPU, builds alternating): 1/16 on the
// polynomial is 6-7% faster than none, 2/16 and 3/16 sit between, and 5/16
// is slower than none: past a small share the polynomial's extra FMA/ALU
// instructions cost more issue slots (and power; the kernels run
// power-capped) than the MUFU time they free.
constexpr uint32_t kEncPolyPairs = 0x0001u;

template <int D, int NHALF, int NS, int PREC = 0>
struct EncodeCfg {
  using G = TileGeom<D>;
  static_assert(PREC == 0 || D <= 64, "split precision needs the split accumulators (D <= 64)");
  static constexpr bool kPSplit = PREC >= 1;  // P as hi + lo
  static constexpr int kQParts = PREC == 2 ? 2 : 1;  // Q as hi (+ lo)
  // D <= 64: each column-half group accumulates its own O with its own
  // reference (no exchange of row maxima); D = 128: the two groups of a slot
  // share one O and agree on the reference through shared memory.
  static constexpr bool kSplitO = D <= 64;
  static constexpr int kAccPerSlot = kSplitO ? 2 : 1;
  static constexpr int kProducerWarp = 16;
  static constexpr int kIssuerWarp = 17;  // + slot
  static constexpr int kThreads = 32 * 19;
  static constexpr uint32_t kColO = 4 * kEncTile;
  static constexpr uint32_t kColQ = kColO + 2 * kAccPerSlot * D;
  // Q in TMEM (TS Q.K^T) when it fits beside S and O, else in shared memory (SS)
  static constexpr bool kQTmem = kColQ + kQParts * D <= 512;
  static constexpr int kQHalfBytes = kQTmem ? 0 : G::bytes(kLatRows);
  static constexpr int kTileBytes = G::bytes(kEncTile);
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kOffQ = 0;  // [part][half] blocks of kQHalfBytes
  static constexpr int kOffStages = kQParts * NHALF * kQHalfBytes;
  static constexpr int kOffBars = kOffStages + NS * kStageBytes;
  // full[NS], empty[NS], q_ready, S_full[4], P_full[4], pv_done[2], O_final[2], drain
  static constexpr int kNumBars = 2 * NS + 14;
  static constexpr int kOffXM = kOffBars + 8 * kNumBars;            // float [2 parity][2 slot][2 half][128]
  static constexpr int kOffML = kOffXM + 2 * 2 * 2 * kLatRows * 4;  // float2 [2 slot][2 half][128]
  static constexpr int kOffMisc = kOffML + 2 * 2 * kLatRows * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + slack for 1024-B alignment
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kColQ <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  // An issuer at local tile i waits for the stage of local tile i + 2 (tile
  // + 2 or + 4), free once the tile before i is released.
  static_assert(NS >= (NHALF == 2 ? 2 : 4) + 1, "ring too shallow for the look-ahead");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16(kLatRows, kEncTile, 0, 0);
  static constexpr uint32_t kIdescPV = ptx::idesc_bf16(kLatRows, D, 0, 1);
  __host__ __device__ static constexpr uint32_t col_s(int s, int j) { return (2 * s + j) * kEncTile; }
  // accumulator of (slot s, column half c): shared by both halves unless kSplitO
  __host__ __device__ static constexpr uint32_t col_o(int s, int c) {
    return kColO + (kSplitO ? 2 * s + c : s) * D;
  }
  // Q of slot s in TMEM: part 0 (hi) then part 1 (lo), each NHALF x D / 2 columns
  __host__ __device__ static constexpr uint32_t col_q(int s, int part = 0) {
    return kColQ + part * NHALF * (D / 2) + (NHALF == 2 ? s : 0) * (D / 2);
  }
};

// The low part of a bf16 pair: bf16(e - hi) for each half, hi = the pair
// pack_bf16 rounded e to (e - hi is exact in fp32).
__device__ __forceinline__ uint32_t bf16_pair_residual(uint64_t e, uint32_t hi) {
  const uint64_t h = ptx::f2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u));
  const uint64_t r = ptx::fma2(h, ptx::f2(-1.f, -1.f), e);
  float r0, r1;
  ptx::f2_split(r, r0, r1);
  return ptx::pack_bf16(r0, r1);
}

// P = 2^(x log2e - nref) for the 32 scores of one half-row, packed to bf16
// pairs and stored into 16 TMEM columns at tP; returns the fp32 sum.
// RAGGED (a tile past the end of the tokens, masked columns at -inf): every
// exponential on MUFU, and masked columns give exactly 0.
// PSPLIT: P on MUFU only, its low parts (P - bf16(P)) into the 16 columns
// after tP.
template <bool RAGGED, bool PSPLIT = false>
__device__ __forceinline__ float encode_exp_store(const float* x, float nref, uint32_t tP) {
  // pairs of columns as packed fp32 (f32x2): x log2e - nref, the polynomial
  // exponentials and the running sums take one instruction per pair
  const uint64_t kL2 = ptx::f2(kLog2e, kLog2e);
  const uint64_t nn = ptx::f2(-nref, -nref);
  uint64_t ps[2] = {0ull, 0ull};  // two independent packed partial sums (+0.0f pairs)
#pragma unroll
  for (int c0 = 0; c0 < 32; c0 += 16) {
    uint32_t p[8], pl[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + 2 * u;
      const uint64_t a = ptx::fma2(ptx::f2(x[c], x[c + 1]), kL2, nn);
      uint64_t e;
      if (!RAGGED && !PSPLIT && ((kEncPolyPairs >> ((c / 2) & 15)) & 1u)) {
        e = exp2_poly3_x2(a);
      } else {
        float a0, a1;
        ptx::f2_split(a, a0, a1);
        float p0 = ptx::ex2(a0), p1 = ptx::ex2(a1);
        if (RAGGED) {  // a half-row may be fully masked with no reference yet (-inf - -inf)
          p0 = x[c] == -INFINITY ? 0.f : p0;
          p1 = x[c + 1] == -INFINITY ? 0.f : p1;
        }
        e = ptx::f2(p0, p1);
      }
      ps[u & 1] = ptx::add2(ps[u & 1], e);
      float e0, e1;
      ptx::f2_split(e, e0, e1);
      p[u] = ptx::pack_bf16(e0, e1);
      if constexpr (PSPLIT) pl[u] = bf16_pair_residual(e, p[u]);
    }
    ptx::tmem_st8(tP + c0 / 2, p);
    if constexpr (PSPLIT) ptx::tmem_st8(tP + 16 + c0 / 2, pl);
  }
  float s0, s1, s2, s3;
  ptx::f2_split(ps[0], s0, s1);
  ptx::f2_split(ps[1], s2, s3);
  return (s0 + s1) + (s2 + s3);
}

// P = 2^(x log2e - nref) for the 32 scores of one full half-row, packed to
// bf16 pairs in p[16]; returns the fp32 sum.  Used against a reference that
// may sit below the half-row's max: the polynomial's input is clamped at 64
// (a result of at most 2^64), so that a score far above the reference shows
// up in the sum (MUFU gives +inf there) instead of wrapping the exponent
// field.  PSPLIT: on MUFU only, with the low parts in pl[16].
template <bool PSPLIT = false>
__device__ __forceinline__ float encode_exp_pack(const float* x, float nref, uint32_t* p, uint32_t* pl) {
  const uint64_t kL2 = ptx::f2(kLog2e, kLog2e);
  const uint64_t nn = ptx::f2(-nref, -nref);
  uint64_t ps[2] = {0ull, 0ull};
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const int c = 2 * u;
    const uint64_t a = ptx::fma2(ptx::f2(x[c], x[c + 1]), kL2, nn);
    uint64_t e;
    float a0, a1;
    ptx::f2_split(a, a0, a1);
    if (!PSPLIT && ((kEncPolyPairs >> (u & 15)) & 1u)) {
      e = exp2_poly3_x2(ptx::f2(fminf(a0, 64.f), fminf(a1, 64.f)));
    } else {
      e = ptx::f2(ptx::ex2(a0), ptx::ex2(a1));
    }
    ps[u & 1] = ptx::add2(ps[u & 1], e);
    float e0, e1;
    ptx::f2_split(e, e0, e1);
    p[u] = ptx::pack_bf16(e0, e1);
    if constexpr (PSPLIT) pl[u] = bf16_pair_residual(e, p[u]);
  }
  float s0, s1, s2, s3;
  ptx::f2_split(ps[0], s0, s1);
  ptx::f2_split(ps[1], s2, s3);
  return (s0 + s1) + (s2 + s3);
}

template <int D, int NHALF, int NS, int PREC>
__global__ void __launch_bounds__(EncodeCfg<D, NHALF, NS, PREC>::kThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmQlo,
                     const EncodeArgs args) {
  using C = EncodeCfg<D, NHALF, NS, PREC>;
  using G = typename C::G;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + NS;
  uint64_t* q_ready = bars + 2 * NS;
  uint64_t* S_full = bars + 2 * NS + 1;    // [2 slot + buffer]
  uint64_t* P_full = bars + 2 * NS + 5;    // [2 slot + buffer]
  uint64_t* pv_done = bars + 2 * NS + 9;   // [slot]
  uint64_t* O_final = bars + 2 * NS + 11;  // [slot]
  uint64_t* drain = bars + 2 * NS + 13;
  float* s_xm = reinterpret_cast<float*>(smem + C::kOffXM);
  float2* s_ml = reinterpret_cast<float2*>(smem + C::kOffML);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int bh = blockIdx.y;
  const int qidx = args.q_batched ? bh : bh % args.H;
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
    // Q in TMEM: one arrival per softmax warp that stores a part of it
    ptx::mbar_init(q_ready, C::kQTmem ? 4 * (NHALF == 2 ? 2 : 1) * (D >= 32 ? 2 : 1) : 1);
    for (int i = 0; i < 4; ++i) {
      ptx::mbar_init(&S_full[i], 1);
      ptx::mbar_init(&P_full[i], 8);  // one arrival per warp of the slot's two groups
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&pv_done[i], 1);
      ptx::mbar_init(&O_final[i], 1);
    }
    ptx::mbar_init(drain, 64);  // one commit per lane of the two issuer warps
    *s_abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == C::kProducerWarp) {
    ptx::tmem_alloc(s_tmem, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t sbase = ptx::smem_u32(smem);
  // Launched with programmatic serialisation (the routing encode of a mixer
  // call), this kernel may start while the kernel before it finishes: every
  // thread but the producer's waits for it here; the producer first
  // prefetches K/V stages (inputs of the call, which no earlier kernel of it
  // writes) and waits before it loads Q.
  if (warp != C::kProducerWarp || lane != 0) ptx::grid_dep_wait();

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmK);
      ptx::prefetch_tmap(&tmV);
      const uint64_t pol = ptx::policy_evict_first();
      int issued = 0;
      auto load_stage = [&](int t) {
        const int st = t % NS;
        uint8_t* sk = smem + C::kOffStages + st * C::kStageBytes;
        uint8_t* sv = sk + C::kTileBytes;
        const int tok = (tile0 + t) * kEncTile;
        ptx::mbar_arrive_expect_tx(&full[st], C::kStageBytes);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sk + b * kEncTile * 128, &tmK, &full[st], b * 64, tok, bh, pol);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sv + b * kEncTile * 128, &tmV, &full[st], b * 64, tok, bh, pol);
        issued = t + 1;
      };
      for (int t = 0; t < NS && t < T; ++t) load_stage(t);
      ptx::grid_dep_wait();
      if constexpr (!C::kQTmem) {
        ptx::prefetch_tmap(&tmQ);
        if constexpr (C::kQParts == 2) ptx::prefetch_tmap(&tmQlo);
        ptx::mbar_arrive_expect_tx(q_ready, C::kQParts * NHALF * C::kQHalfBytes);
        for (int part = 0; part < C::kQParts; ++part)
          for (int h = 0; h < NHALF; ++h)
            for (int b = 0; b < G::kBlocks; ++b)
              ptx::tma_load_3d(smem + C::kOffQ + (part * NHALF + h) * C::kQHalfBytes + b * kLatRows * 128,
                               part ? &tmQlo : &tmQ, q_ready, b * 64, h * kLatRows, qidx);
      }
      for (int t = issued; t < T; ++t) {
        if (t >= NS && !ptx::mbar_wait(&empty[t % NS], ((t / NS) - 1) & 1, s_abort, args.wait_ns)) {
          record_error(args.status, kErrTimeout, kSiteEncProducer);
          *s_abort = 1;
          break;
        }
        load_stage(t);
      }
      // this CTA's loads are all issued: the next kernel of the stream may start
      ptx::grid_dep_launch();
      // Every load issued must land before the CTA may exit (matters on the abort path only).
      if constexpr (!C::kQTmem) ptx::mbar_wait_drain(q_ready, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        ptx::mbar_wait_drain(&full[t % NS], (t / NS) & 1);
    }
  } else if (warp >= C::kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuers
    // The whole warp runs the loop (waits are warp-wide); one elected lane
    // issues each batch of MMAs and the commits that track them.
    const int s = warp - C::kIssuerWarp;
    const int count = count_of(s);
    const uint64_t dK0 = G::kmajor(sbase + C::kOffStages, kEncTile, 0);
    const uint64_t dV0 = G::mnmajor(sbase + C::kOffStages + C::kTileBytes, kEncTile, 0);
    const uint64_t dQ = G::kmajor(sbase + C::kOffQ + (NHALF == 2 ? s : 0) * C::kQHalfBytes, kLatRows, 0);
    const uint32_t tQ = tmem + C::col_q(s);
    // the low parts of Q (split precision): NHALF half blocks further in smem,
    // or their own TMEM columns
    constexpr uint32_t kQloSmemStep = static_cast<uint32_t>(NHALF * C::kQHalfBytes) >> 4;
    const uint32_t tQlo = tmem + C::col_q(s, C::kQParts - 1);
    auto wait_stage = [&](int t) -> bool {
      return ptx::mbar_wait(&full[t % NS], (t / NS) & 1, s_abort, args.wait_ns);
    };
    auto issue_qk = [&](int i) {
      const int t = tile_of(s, i);
      const uint32_t tS = tmem + C::col_s(s, i & 1);
      const uint64_t dK = dK0 + static_cast<uint32_t>((t % NS) * (C::kStageBytes >> 4));
#pragma unroll
      for (int part = 0; part < C::kQParts; ++part) {
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t acc = (k > 0 || part > 0) ? 1u : 0u;
          if constexpr (C::kQTmem)
            ptx::mma_ts(tS, (part ? tQlo : tQ) + k * 8, dK + G::kmajor_step(kEncTile, k), C::kIdescQK, acc);
          else
            ptx::mma_ss(tS, dQ + part * kQloSmemStep + G::kmajor_step(kLatRows, k), dK + G::kmajor_step(kEncTile, k),
                        C::kIdescQK, acc);
        }
      }
      ptx::mma_commit(&S_full[2 * s + (i & 1)]);
    };
    bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(q_ready, 0, s_abort, args.wait_ns));
    // Slot 1 starts once slot 0's first P is stored, so that the two slots'
    // softmax phases interleave instead of running in step.
    if (s == 1 && count_of(0) > 0)
      ok = ok && __all_sync(0xffffffffu, ptx::mbar_wait(&P_full[0], 0, s_abort, args.wait_ns));
    for (int i = 0; ok && i < 2 && i < count; ++i) {
      ok = __all_sync(0xffffffffu, wait_stage(tile_of(s, i)));
      if (ok) {
        ptx::tc_fence_after();
        if (ptx::elect_one()) issue_qk(i);
        __syncwarp();
      }
    }
    for (int i = 0; ok && i < count; ++i) {
      const int t = tile_of(s, i);
      // every wait before the MMAs: a wait after them would stall until they complete
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(&P_full[2 * s + (i & 1)], (i >> 1) & 1, s_abort, args.wait_ns) &&
                                       (i + 2 >= count || wait_stage(tile_of(s, i + 2))));
      if (!ok) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
        const uint32_t tP = tmem + C::col_s(s, i & 1);
        const uint64_t dV = dV0 + static_cast<uint32_t>((t % NS) * (C::kStageBytes >> 4));
        // K steps 0-1 carry the tokens of column half 0, steps 2-3 those of half 1
        // (split precision: each step once with P_hi, once with P_lo 16 columns on)
#pragma unroll
        for (int kk = 0; kk < kEncTile / 16; ++kk) {
          const int cu = kk / 2;
#pragma unroll
          for (int part = 0; part < (C::kPSplit ? 2 : 1); ++part) {
            const bool acc = i > 0 || (C::kSplitO ? (kk & 1) : kk) > 0 || part > 0;
            ptx::mma_ts(tmem + C::col_o(s, cu), tP + cu * 32 + part * 16 + (kk & 1) * 8, dV + G::mnmajor_step(kk),
                        C::kIdescPV, acc ? 1u : 0u);
          }
        }
        ptx::mma_commit(&empty[t % NS]);
        ptx::mma_commit(&pv_done[s]);
        if (i + 2 < count) issue_qk(i + 2);  // into the buffer P(i) came from: after its P.V in issue order
        if (i + 1 == count) ptx::mma_commit(&O_final[s]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      record_error(args.status, kErrTimeout, kSiteEncMma);
      *s_abort = 1;
    }
    // Drain: every lane commits (a lane that issued nothing arrives at once),
    // so every MMA issued completes before TMEM is released.
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
  } else {
    // ------------------------------------------------------------ softmax groups
    const int g = warp >> 2;               // group
    const int s = g >> 1;                  // slot
    const int c = g & 1;                   // column half
    const int r = (warp & 3) * 32 + lane;  // TMEM lane = latent row within the half
    const int m = (NHALF == 2 ? s : 0) * kLatRows + r;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int count = count_of(s);

    if constexpr (C::kQTmem) {
      // Q row m into TMEM as bf16 pairs; group c stores its half of the columns.
      constexpr int kQCols = D / 2;  // 32-bit columns per row
      constexpr int kPart = kQCols >= 16 ? kQCols / 2 : kQCols;
      if ((NHALF == 2 || s == 0) && (kQCols >= 16 || c == 0)) {
        uint32_t qv[kPart];
        const int col0 = kQCols >= 16 ? c * kPart : 0;
        if (m < args.M) {
          const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(args.Q) +
                                                            (static_cast<size_t>(qidx) * args.M + m) * D) +
                             col0 / 4;
#pragma unroll
          for (int z = 0; z < kPart / 4; ++z) {
            const uint4 v = src[z];
            qv[4 * z] = v.x;
            qv[4 * z + 1] = v.y;
            qv[4 * z + 2] = v.z;
            qv[4 * z + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int z = 0; z < kPart; ++z) qv[z] = 0u;
        }
        const uint32_t ta = tmem + lane_off + C::col_q(s) + col0;
        if constexpr (kPart == 16) ptx::tmem_st16(ta, qv); else ptx::tmem_st8(ta, qv);
        if constexpr (C::kQParts == 2) {
          // the low parts of the same row into their own columns
          if (m < args.M) {
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(args.Q_lo) +
                                                              (static_cast<size_t>(qidx) * args.M + m) * D) +
                               col0 / 4;
#pragma unroll
            for (int z = 0; z < kPart / 4; ++z) {
              const uint4 v = src[z];
              qv[4 * z] = v.x;
              qv[4 * z + 1] = v.y;
              qv[4 * z + 2] = v.z;
              qv[4 * z + 3] = v.w;
            }
          }
          const uint32_t tl = tmem + lane_off + C::col_q(s, 1) + col0;
          if constexpr (kPart == 16) ptx::tmem_st16(tl, qv); else ptx::tmem_st8(tl, qv);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(q_ready);
      }
    }

    float mref = -INFINITY, l = 0.f;  // reference max (log2 domain), running sum of this half-row
    bool ok = true;
    const int bar_id = 1 + s;  // named barrier of the slot's two groups (shared O only)
    constexpr int kOCols = C::kSplitO ? D : D / 2;  // O columns this group rescales
    const uint32_t tOwn = tmem + lane_off + C::col_o(s, c) + (C::kSplitO ? 0 : c * (D / 2));
    for (int i = 0; i < count; ++i) {
      const int t = tile_of(s, i);
      const int j = i & 1;
      const uint32_t tS = tmem + lane_off + C::col_s(s, j);
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&S_full[2 * s + j], (i >> 1) & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      float x[32];
      ptx::tmem_ld32(tS + 32 * c, x);
      ptx::tmem_wait_ld();
      const int valid = args.N - (tile0 + t) * kEncTile - 32 * c;
      if (valid < 32) {
#pragma unroll
        for (int z = 0; z < 32; ++z)
          if (z >= valid) x[z] = -INFINITY;
      }
      // Past the first tile the reference is usually high enough: take the
      // exponentials against it without the half-row max, and fall back to the
      // max below only if some score of the tile sits far above it (a sum
      // above 2^32, or inf).  Split accumulators only: with a shared O the two
      // groups must take the same path.
      bool done = false;
      if (C::kSplitO && i > 0 && valid >= 32) {
        uint32_t p[16], pl[16];
        const float lt = encode_exp_pack<C::kPSplit>(x, mref, p, pl);
        if (__all_sync(0xffffffffu, lt <= 4294967296.f)) {
          ptx::tmem_st16(tS + 32 * c, p);
          if constexpr (C::kPSplit) ptx::tmem_st16(tS + 32 * c + 16, pl);
          l += lt;
          done = true;
        }
      }
      if (!done) {
        // half-row max as 8 independent 3-input chains
        float pm[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = fmaxf(x[2 * u], x[2 * u + 1]);
#pragma unroll
        for (int u = 0; u < 8; ++u) pm[u] = ptx::max3(pm[u], x[16 + 2 * u], x[17 + 2 * u]);
        float mx = ptx::max3(ptx::max3(pm[0], pm[1], pm[2]), ptx::max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        if constexpr (!C::kSplitO) {
          // shared O: agree on the row max with the other group of the slot
          // (buffers alternate by tile parity, so a fast group cannot overwrite
          // a value not yet read); after the barrier both groups have read
          // their scores and P may overwrite S
          float* xm = s_xm + ((j * 2 + s) * 2) * kLatRows;
          xm[c * kLatRows + r] = mx;
          asm volatile("bar.sync %0, 256;" ::"r"(bar_id) : "memory");
          mx = fmaxf(mx, xm[(c ^ 1) * kLatRows + r]);
        }
        mx *= kLog2e;
        const bool need = mx > mref + 8.f;
        const float nref = need ? mx : mref;
        // 0 on the first tile; 1 while a fully masked half-row has no reference
        const float alpha = nref == mref ? 1.f : ptx::ex2(mref - nref);
        mref = nref;
        // P overwrites the first 16 of this group's own 32 score columns
        const float lt = valid < 32 ? encode_exp_store<true, C::kPSplit>(x, nref, tS + 32 * c)
                                    : encode_exp_store<false, C::kPSplit>(x, nref, tS + 32 * c);
        l = fmaf(l, alpha, lt);
        // Rare: the reference moved, so rescale this group's part of O, once the
        // previous P.V (issued after P(i - 1)) has completed; the next one waits
        // for P_full.
        if (i > 0 && __any_sync(0xffffffffu, need)) {
          if (!__all_sync(0xffffffffu, ptx::mbar_wait(&pv_done[s], (i - 1) & 1, s_abort, args.wait_ns))) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          constexpr int kChunk = kOCols < 32 ? kOCols : 32;
#pragma unroll
          for (int z0 = 0; z0 < kOCols; z0 += kChunk) {
            float o[kChunk];
            const uint32_t ta = tOwn + z0;
            if constexpr (kChunk == 32) ptx::tmem_ld32(ta, o); else if constexpr (kChunk == 16) ptx::tmem_ld16(ta, o); else ptx::tmem_ld8(ta, o);
            ptx::tmem_wait_ld();
            uint32_t u[kChunk];
#pragma unroll
            for (int z = 0; z < kChunk; ++z) u[z] = __float_as_uint(o[z] * alpha);
            if constexpr (kChunk == 32) ptx::tmem_st32(ta, u); else if constexpr (kChunk == 16) ptx::tmem_st16(ta, u); else ptx::tmem_st8(ta, u);
          }
        }
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&P_full[2 * s + j]);
    }
    if (!ok) {
      record_error(args.status, kErrTimeout, kSiteEncSoftmax);
      *s_abort = 1;
    }

    // ---------------------------------------------------------- epilogue
    // Every group publishes (mref, l); the writer groups (both groups of a
    // slot when M > 128, slot 0's when M <= 128) fold the accumulators that
    // cover their rows into one partial, group c writing columns
    // [c D / 2, +D / 2).
    s_ml[(s * 2 + c) * kLatRows + r] = make_float2(count > 0 ? mref : -INFINITY, count > 0 ? l : 0.f);
    __syncwarp();
    asm volatile("bar.sync 3, 512;" ::: "memory");  // all four groups
    const bool writer = NHALF == 2 || s == 0;
    if (writer && ok) {
      constexpr int kSlotsIn = NHALF == 2 ? 1 : 2;      // slots folded into the partial
      constexpr int kAcc = kSlotsIn * C::kAccPerSlot;  // accumulators folded
      float w[kAcc], ms = -INFINITY, lsum = 0.f;
#pragma unroll
      for (int u = 0; u < kSlotsIn; ++u) {
        const int su = NHALF == 2 ? s : u;
        if (count_of(su) == 0) continue;  // uniform
#pragma unroll
        for (int cu = 0; cu < C::kAccPerSlot; ++cu) ms = fmaxf(ms, s_ml[(su * 2 + cu) * kLatRows + r].x);
        ok = ok && __all_sync(0xffffffffu, ptx::mbar_wait(&O_final[su], 0, s_abort, args.wait_ns));
      }
#pragma unroll
      for (int u = 0; u < kSlotsIn; ++u) {
        const int su = NHALF == 2 ? s : u;
        const float2 a0 = s_ml[(su * 2) * kLatRows + r], a1 = s_ml[(su * 2 + 1) * kLatRows + r];
        if constexpr (C::kSplitO) {
          w[2 * u] = count_of(su) > 0 ? ptx::ex2(a0.x - ms) : 0.f;
          w[2 * u + 1] = count_of(su) > 0 ? ptx::ex2(a1.x - ms) : 0.f;
          lsum = fmaf(w[2 * u], a0.y, fmaf(w[2 * u + 1], a1.y, lsum));
        } else {
          // one accumulator, one reference per slot; both halves' sums
          w[u] = count_of(su) > 0 ? ptx::ex2(a0.x - ms) : 0.f;
          lsum = fmaf(w[u], a0.y + a1.y, lsum);
        }
      }
      if (ok) {
        ptx::tc_fence_after();
        const size_t row = (static_cast<size_t>(bh) * args.P + split) * args.M + m;
        constexpr int kHalfD = D / 2;
        constexpr int kChunk = kHalfD < 32 ? kHalfD : 32;
        float4* dst = reinterpret_cast<float4*>(args.O_part + row * D + c * kHalfD);
#pragma unroll
        for (int z0 = 0; z0 < kHalfD; z0 += kChunk) {
          float acc[kChunk];
#pragma unroll
          for (int z = 0; z < kChunk; ++z) acc[z] = 0.f;
#pragma unroll
          for (int a = 0; a < kAcc; ++a) {
            const int su = NHALF == 2 ? s : a / C::kAccPerSlot;
            if (count_of(su) == 0) continue;  // its accumulator was never written
            float o[kChunk];
            const uint32_t ta = tmem + lane_off + C::col_o(su, a % C::kAccPerSlot) + c * kHalfD + z0;
            if constexpr (kChunk == 32) ptx::tmem_ld32(ta, o); else if constexpr (kChunk == 16) ptx::tmem_ld16(ta, o); else ptx::tmem_ld8(ta, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int z = 0; z < kChunk; ++z) acc[z] = fmaf(w[a], o[z], acc[z]);
          }
          if (m < args.M) {
            if (args.direct) {
              encode_store_direct<kChunk>(args, row * D + c * kHalfD + z0, acc, lsum);
            } else {
#pragma unroll
              for (int z = 0; z < kChunk / 4; ++z)
                dst[z0 / 4 + z] = make_float4(acc[4 * z], acc[4 * z + 1], acc[4 * z + 2], acc[4 * z + 3]);
            }
          }
        }
        if (m < args.M && c == 0) {
          if (args.direct) {
            constexpr float kLn2 = 0.6931471805599453f;
            if (args.lse_out) args.lse_out[row] = lsum > 0.f ? (ms + log2f(lsum)) * kLn2 : -INFINITY;
          } else {
            args.m_part[row] = ms;
            args.l_part[row] = lsum;
          }
        }
      } else {
        record_error(args.status, kErrTimeout, kSiteEncSoftmax);
        *s_abort = 1;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kProducerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace flare
