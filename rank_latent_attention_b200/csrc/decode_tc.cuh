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
// memory, and a contiguous run of 128-token tiles, taken alternately by two
// slots.
//   warps 0-15   four softmax warpgroups (slot s, latent half c): thread r of
//                group (s, c) owns token r of the slot's tiles and latents
//                [c MP / 2, (c + 1) MP / 2)
//   warp 16      TMA producer: Q and Z once, then K tiles into an NS ring;
//                also allocates TMEM
//   warps 17-18  tcgen05.mma issuers, one warp per slot
// Per tile of a slot: S = K_tile Q^T (128 x MP fp32 in TMEM); each group takes
// the max over its half-row, the two groups exchange it through shared
// memory (named barrier), each writes P = 2^(s log2e - max) as bf16 pairs
// into its own score columns and keeps its half of the row sum; then
// O = P Z (128 x D) in TMEM, and each group scales half of O's columns by
// 1 / (sum of both halves) and stores them as bf16 rows of Y.  S of the
// slot's next tile is computed as soon as its columns are free: the latent
// half whose columns hold no O with P.V, the other once O has been read.
// The slots take turns at the exponentials, so one slot's softmax overlaps
// the other's MMAs and epilogue.
//
// The issuer warps run their loop as a whole and issue under elect.sync,
// which keeps the MMA operands warp-uniform.  The softmax arithmetic runs on
// packed fp32 pairs (f32x2); the column pairs in kDecPolyPairs would take
// their exponentials from exp2_poly3 (FMA pipe) instead of MUFU.
//
// TMEM: slot s owns columns [256 s, 256 s + 256): S at [0, MP); P of group 0
// at [0, MP / 4) (latent pairs in order, written over scores already read);
// P of group 1 at [3 MP / 4, MP) (its chunks processed last to first, so each
// P chunk lands on scores already read); O at kColO: [MP / 4, MP / 4 + D) for
// MP = 256 (free once both groups have stored P), [128, 128 + D) for MP = 128.
//
// Split precision (PREC = 1).  Each rounded MMA operand is carried as a pair
// hi + lo of 16-bit numbers (hi = round(x), lo = round(x - hi)), and each
// product takes one MMA per part:
//   S = K Q_hi^T + K Q_lo^T          Q_dyn as a bf16 pair (K is exact bf16);
//   O = P Z_hi + P Z_lo              P and Z in fp16, on kind::f16 with fp16
//                                    operands.
// P lies in [0, 1] (the row max is subtracted exactly), so fp16 holds it to
// 2^-11 relative, 8x finer than bf16, in the same 16 bits of TMEM: the slot
// layout above is unchanged.  Z is read as fp32 from global memory; each CTA
// scales its head's Z by 2^-e, with e chosen from the head's max|Z| so that
// the scaled values lie below 2^15 (inside fp16's range, whatever the inputs'
// range), writes the fp16 pair into shared memory in the swizzled layout the
// tensor map would have produced, and multiplies Y by 2^e in the epilogue.
// Y is written in fp32 (16-byte stores of four floats).
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"

namespace flare {

struct DecodeArgs {
  int N;
  int M;
  int q_batched;  // Q indexed by bh (1) or h = bh % H (0)
  int H;
  int splits;
  int tiles;
  void* Y;  // [BH][N][D]: bf16, or fp32 with split precision
  const float* Zf;  // split precision: Z as fp32 [BH][M][D] (the bf16 Z map is unused)
  int* status;
  unsigned long long wait_ns;
};

// Column pairs (bit j: pair j of each 16) whose exponentials go to
// exp2_poly3 in the decode softmax: none (A/B measured: 1/16 makes no
// difference, 2/16 is slower, 5/16 much slower).
constexpr uint32_t kDecPolyPairs = 0x0000u;

template <int D, int MP, int NS, int PREC = 0>
struct DecodeCfg {
  using G = TileGeom<D>;
  static_assert(MP == 128 || MP == 256, "padded latent count");
  static constexpr int kLatParts = PREC ? 2 : 1;  // Q_dyn and Z as hi (+ lo)
  static constexpr int kHalf = MP / 2;      // latents per group
  static constexpr int kChunks = kHalf / 32;  // 32-latent chunks per group
  static constexpr int kProducerWarp = 16;
  static constexpr int kIssuerWarp = 17;  // + slot
  static constexpr int kThreads = 32 * 19;
  static constexpr int kLatBytes = G::bytes(MP);
  static constexpr int kTileBytes = G::bytes(kTileN);
  static constexpr int kOffQ = 0;
  static constexpr int kOffZ = kLatBytes;
  static constexpr int kOffQlo = 2 * kLatBytes;  // split precision only
  static constexpr int kOffZlo = 3 * kLatBytes;
  static constexpr int kOffStages = 2 * kLatParts * kLatBytes;
  static constexpr int kOffBars = kOffStages + NS * kTileBytes;
  // full[NS], empty[NS], qz_full, S_full[2], P_full[2], O_full[2], O_free[2], turn[2], drain
  static constexpr int kNumBars = 2 * NS + 12;
  static constexpr int kOffXM = kOffBars + 8 * kNumBars;  // float [2 slot][2 half][128]: half-row max
  static constexpr int kOffXL = kOffXM + 2 * 2 * 128 * 4;  // float [2 slot][2 half][128]: half-row sum
  static constexpr int kOffMisc = kOffXL + 2 * 2 * 128 * 4;
  static constexpr int kOffRed = kOffMisc + 16;  // float [16]: per-warp max|Z| (split precision)
  static constexpr int kSmemBytes = kOffRed + 64 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kSlotCols = 256;
  static constexpr uint32_t kColP1 = 3 * MP / 4;
  static constexpr uint32_t kColO = MP == 256 ? MP / 4 : 128;
  static_assert(kColO + D <= (MP == 256 ? kColP1 : kSlotCols), "TMEM slot layout");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
  static constexpr uint32_t kIdescQK = ptx::idesc_bf16(kTileN, MP, 0, 0);
  static constexpr uint32_t kIdescQKHalf = ptx::idesc_bf16(kTileN, kLatRows, 0, 0);  // one latent half
  static constexpr uint32_t kIdescPV = PREC ? ptx::idesc_f16(kTileN, D, 0, 1) : ptx::idesc_bf16(kTileN, D, 0, 1);
  // qz_full: the producer's expect_tx arrival, plus (split precision) one per
  // softmax warp once its part of the fp16 Z is in shared memory
  static constexpr int kQzArrivals = PREC ? 1 + 16 : 1;
  // TMEM column (within the slot) of P for latents [16 kk, +16): the PV K step kk
  __host__ __device__ static constexpr uint32_t col_pk(int kk) {
    return kk < MP / 32 ? 8 * kk : kColP1 + 8 * (kk - MP / 32);
  }
};

// P for one 32-latent chunk of a row: 2^(x log2e - mref) for the valid
// columns (16-column groups at or past M give P = 0), packed to bf16 pairs
// into 16 TMEM columns at tP; returns the fp32 sum.
template <int MP, bool F16P = false>
__device__ __forceinline__ float decode_exp_chunk(const float* x, float mref, int col0, int M, uint32_t tP) {
  const uint64_t kL2 = ptx::f2(kLog2e, kLog2e);
  const uint64_t nn = ptx::f2(-mref, -mref);
  uint64_t ps[2] = {0ull, 0ull};
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    uint32_t p[8];
    if (col0 + 16 * g < M) {
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = 16 * g + 2 * u;
        const uint64_t a = ptx::fma2(ptx::f2(x[c], x[c + 1]), kL2, nn);
        uint64_t e;
        if ((kDecPolyPairs >> (u + 8 * g)) & 1u) {
          e = exp2_poly3_x2(a);
        } else {
          float a0, a1;
          ptx::f2_split(a, a0, a1);
          e = ptx::f2(ptx::ex2(a0), ptx::ex2(a1));
        }
        ps[u & 1] = ptx::add2(ps[u & 1], e);
        float e0, e1;
        ptx::f2_split(e, e0, e1);
        p[u] = F16P ? ptx::pack_f16(e0, e1) : ptx::pack_bf16(e0, e1);
      }
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) p[u] = 0u;
    }
    ptx::tmem_st8(tP + 8 * g, p);
  }
  float s0, s1, s2, s3;
  ptx::f2_split(ps[0], s0, s1);
  ptx::f2_split(ps[1], s2, s3);
  return (s0 + s1) + (s2 + s3);
}

// Split precision: the head's fp32 Z [M][D] (rows past M as zeros), scaled by
// 2^-e with e = the exponent that puts the head's max|Z| in [2^14, 2^15),
// into shared memory as an fp16 pair (hi at kOffZ, lo at kOffZlo) in the
// layout a TMA load with the tile's swizzle produces (16-byte chunks of a row
// permuted by address bits 7 and up); run by the 512 softmax threads (tid),
// returns 2^e.  Every thread fences its stores for the tensor core's reads.
template <int D, int MP, int NS, int PREC>
__device__ __forceinline__ float stage_z_f16(const DecodeArgs& args, uint8_t* smem, int tid) {
  using C = DecodeCfg<D, MP, NS, PREC>;
  using G = typename C::G;
  static_assert(D <= 64, "one column block");
  constexpr int kRowChunks = D / 8;  // 16-byte chunks of 8 fp16 per row
  constexpr int kChunks = MP * kRowChunks;
  constexpr uint32_t kSwzMask = G::kSwizzle == 2u ? 7u : (G::kSwizzle == 4u ? 3u : 1u);  // 128 / 64 / 32 B
  float* red = reinterpret_cast<float*>(smem + C::kOffRed);
  const float* Zh = args.Zf + static_cast<size_t>(blockIdx.y) * args.M * D;
  float mx = 0.f;
  for (int q = tid; q < kChunks; q += 512) {
    const int row = q / kRowChunks;
    if (row < args.M) {
      const float4* src = reinterpret_cast<const float4*>(Zh + static_cast<size_t>(row) * D + (q % kRowChunks) * 8);
      const float4 a = src[0], b = src[1];
      mx = fmaxf(mx, ptx::max3(ptx::max3(fabsf(a.x), fabsf(a.y), fabsf(a.z)), ptx::max3(fabsf(a.w), fabsf(b.x), fabsf(b.y)),
                               fmaxf(fabsf(b.z), fabsf(b.w))));
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  asm volatile("bar.sync 5, 512;" ::: "memory");
#pragma unroll
  for (int w = 0; w < 16; ++w) mx = fmaxf(mx, red[w]);
  int e = 0;
  if (mx > 0.f && mx <= 3.4e38f) {
    int ex;
    frexpf(mx, &ex);  // mx = f 2^ex, f in [1/2, 1)
    e = ex - 15;
  }
  const float down = ldexpf(1.f, -e);
  for (int q = tid; q < kChunks; q += 512) {
    const int row = q / kRowChunks, ch = q % kRowChunks;
    float v[8];
    if (row < args.M) {
      const float4* src = reinterpret_cast<const float4*>(Zh + static_cast<size_t>(row) * D + ch * 8);
      const float4 a = src[0], b = src[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int z = 0; z < 8; ++z) v[z] = 0.f;
    }
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int z = 0; z < 4; ++z) {
      const float a = v[2 * z] * down, b = v[2 * z + 1] * down;
      hi[z] = ptx::pack_f16(a, b);
      const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&hi[z]));
      lo[z] = ptx::pack_f16(a - h.x, b - h.y);
    }
    const uint32_t lin = static_cast<uint32_t>(row * G::kRowBytes + ch * 16);
    const uint32_t off = lin ^ (((lin >> 7) & kSwzMask) << 4);
    *reinterpret_cast<uint4*>(smem + C::kOffZ + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
    *reinterpret_cast<uint4*>(smem + C::kOffZlo + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
  }
  ptx::fence_proxy_async_smem();
  return ldexpf(1.f, e);
}

// The softmax / epilogue loop of one group (slot s, latent half CH).
template <int D, int MP, int NS, int PREC>
struct DecodeGroup {
  using C = DecodeCfg<D, MP, NS, PREC>;
  const DecodeArgs& args;
  uint32_t tmem;
  int warp, lane, s, tile0, T;
  uint64_t *S_full, *P_full, *O_full, *O_free, *turn;
  float* xm;  // [2 half][128] of this slot
  float* xl;
  volatile int* s_abort;
  float zscale;  // 2^e, the factor the fp16 Z was scaled down by (1 without split precision)

  template <int CH>
  __device__ __forceinline__ void run() {
    const int r = (warp & 3) * 32 + lane;  // token row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + s * C::kSlotCols;
    const int count = s == 0 ? (T + 1) / 2 : T / 2;
    const int M = args.M;
    constexpr int kLat0 = CH * C::kHalf;  // first latent (S column) of this group
    bool ok = true;
    for (int i = 0; i < count; ++i) {
      const int t = 2 * i + s;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&S_full[s], i & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      // pass 1: max over this group's valid latents (M is a multiple of 16,
      // so validity is uniform per 16-column group)
      float pm[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) pm[j] = -INFINITY;
#pragma unroll
      for (int k = 0; k < C::kChunks; ++k) {
        float x[32];
        ptx::tmem_ld32(tS + kLat0 + 32 * k, x);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h)
          if (kLat0 + 32 * k + 16 * h < M) {
#pragma unroll
            for (int j = 0; j < 8; ++j) pm[j] = ptx::max3(pm[j], x[16 * h + 2 * j], x[16 * h + 2 * j + 1]);
          }
      }
      // exchange with the other group of the slot: the row max over all latents
      xm[CH * 128 + r] = ptx::max3(ptx::max3(pm[0], pm[1], pm[2]), ptx::max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
      asm volatile("bar.sync %0, 256;" ::"r"(1 + s) : "memory");
      const float mref = fmaxf(xm[r], xm[128 + r]) * kLog2e;
      // The slots take turns at the exponentials (slot 0's tile i, slot 1's
      // tile i, slot 0's tile i + 1, ...): one slot computes while the other
      // slot's P.V, epilogue and next Q.K^T run.
      if ((s == 1 || i > 0) &&
          !__all_sync(0xffffffffu, ptx::mbar_wait(&turn[s], (s == 1 ? i : i - 1) & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      // pass 2: P chunk by chunk (group 1 last to first, see the layout note)
      float l = 0.f;
#pragma unroll
      for (int q = 0; q < C::kChunks; ++q) {
        const int k = CH == 0 ? q : C::kChunks - 1 - q;
        float x[32];
        ptx::tmem_ld32(tS + kLat0 + 32 * k, x);
        ptx::tmem_wait_ld();
        l += decode_exp_chunk<MP, PREC != 0>(x, mref, kLat0 + 32 * k, M, tS + (CH == 0 ? 16 * k : C::kColP1 + 16 * k));
      }
      xl[CH * 128 + r] = l;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&turn[s ^ 1]);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&P_full[s]);

      // epilogue: O = P Z; this group scales columns [CH D / 2, +D / 2)
      if (!__all_sync(0xffffffffu, ptx::mbar_wait(&O_full[s], i & 1, s_abort, args.wait_ns))) {
        ok = false;
        break;
      }
      asm volatile("bar.sync %0, 256;" ::"r"(3 + s) : "memory");  // both halves' sums are in xl
      const float inv = zscale / (xl[r] + xl[128 + r]);
      ptx::tc_fence_after();
      constexpr int kHD = D / 2;
      const uint32_t tO = tS + C::kColO + CH * kHD;
      float o[kHD];
      if constexpr (kHD == 64) {
        ptx::tmem_ld32(tO, o);
        ptx::tmem_ld32(tO + 32, o + 32);
      } else if constexpr (kHD == 32) {
        ptx::tmem_ld32(tO, o);
      } else if constexpr (kHD == 16) {
        ptx::tmem_ld16(tO, o);
      } else {
        ptx::tmem_ld8(tO, o);
      }
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&O_free[s]);

      const long long tok = static_cast<long long>(tile0 + t) * kTileN + r;
      if (tok < args.N) {
        const size_t row = (static_cast<size_t>(blockIdx.y) * args.N + tok) * D + CH * kHD;
        if constexpr (PREC) {
          float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.Y) + row);
#pragma unroll
          for (int z = 0; z < kHD / 4; ++z)
            dst[z] = make_float4(o[4 * z] * inv, o[4 * z + 1] * inv, o[4 * z + 2] * inv, o[4 * z + 3] * inv);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.Y) + row);
#pragma unroll
          for (int z = 0; z < kHD / 8; ++z) {
            uint4 v;
            v.x = ptx::pack_bf16(o[8 * z + 0] * inv, o[8 * z + 1] * inv);
            v.y = ptx::pack_bf16(o[8 * z + 2] * inv, o[8 * z + 3] * inv);
            v.z = ptx::pack_bf16(o[8 * z + 4] * inv, o[8 * z + 5] * inv);
            v.w = ptx::pack_bf16(o[8 * z + 6] * inv, o[8 * z + 7] * inv);
            dst[z] = v;
          }
        }
      }
    }
    if (!ok) {
      record_error(args.status, kErrTimeout, kSiteDecSoftmax);
      *s_abort = 1;
    }
  }
};

template <int D, int MP, int NS, int PREC>
__global__ void __launch_bounds__(DecodeCfg<D, MP, NS, PREC>::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmQlo,
                     const __grid_constant__ CUtensorMap tmZlo, const DecodeArgs args) {
  using C = DecodeCfg<D, MP, NS, PREC>;
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
  uint64_t* turn = bars + 2 * NS + 9;  // [slot]: the other slot has finished its exponentials
  uint64_t* drain = bars + 2 * NS + 11;
  float* s_xm = reinterpret_cast<float*>(smem + C::kOffXM);
  float* s_xl = reinterpret_cast<float*>(smem + C::kOffXL);
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
    ptx::mbar_init(qz_full, C::kQzArrivals);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&S_full[s], 1);
      ptx::mbar_init(&P_full[s], 8);  // one arrival per warp of the slot's two groups
      ptx::mbar_init(&O_full[s], 1);
      ptx::mbar_init(&O_free[s], 8);
      ptx::mbar_init(&turn[s], 8);
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
  // Launched with programmatic serialisation (the decode of a mixer call),
  // this kernel may start while the kernel before it finishes: every thread
  // but the producer's waits for it here; the producer first prefetches K
  // stages (an input of the call) and waits before it loads Q and Z.
  if (warp != C::kProducerWarp || lane != 0) ptx::grid_dep_wait();

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      ptx::prefetch_tmap(&tmK);
      const uint64_t pol = ptx::policy_evict_first();
      int issued = 0;
      auto load_stage = [&](int t) {
        const int st = t % NS;
        uint8_t* sk = smem + C::kOffStages + st * C::kTileBytes;
        ptx::mbar_arrive_expect_tx(&full[st], C::kTileBytes);
        for (int b = 0; b < G::kBlocks; ++b)
          ptx::tma_load_3d_hint(sk + b * kTileN * 128, &tmK, &full[st], b * 64, (tile0 + t) * kTileN, bh, pol);
        issued = t + 1;
      };
      for (int t = 0; t < NS && t < T; ++t) load_stage(t);
      ptx::grid_dep_wait();
      ptx::prefetch_tmap(&tmQ);
      // split precision: Q_hi and Q_lo by TMA, the fp16 Z pair from the softmax warps
      const CUtensorMap* second = PREC ? &tmQlo : &tmZ;
      ptx::prefetch_tmap(second);
      const int qidx = args.q_batched ? bh : bh % args.H;
      ptx::mbar_arrive_expect_tx(qz_full, 2 * C::kLatBytes);
      for (int h = 0; h < MP / kLatRows; ++h)
        for (int b = 0; b < G::kBlocks; ++b) {
          const int off = b * MP * 128 + h * kLatRows * G::kRowBytes;
          ptx::tma_load_3d(smem + C::kOffQ + off, &tmQ, qz_full, b * 64, h * kLatRows, qidx);
          ptx::tma_load_3d(smem + (PREC ? C::kOffQlo : C::kOffZ) + off, second, qz_full, b * 64, h * kLatRows,
                           PREC ? qidx : bh);
        }
      for (int t = issued; t < T; ++t) {
        if (t >= NS && !ptx::mbar_wait(&empty[t % NS], ((t / NS) - 1) & 1, s_abort, args.wait_ns)) {
          record_error(args.status, kErrTimeout, kSiteDecProducer);
          *s_abort = 1;
          break;
        }
        load_stage(t);
      }
      // this CTA's loads are all issued: the next kernel of the stream may start
      ptx::grid_dep_launch();
      ptx::mbar_wait_drain(qz_full, 0);
      for (int t = (issued > NS ? issued - NS : 0); t < issued; ++t)
        ptx::mbar_wait_drain(&full[t % NS], (t / NS) & 1);
    }
  } else if (warp >= C::kIssuerWarp) {
    // ------------------------------------------------------------ MMA issuers (one warp per slot)
    // The whole warp runs the loop (waits are warp-wide); one elected lane
    // issues each batch of MMAs and the commits that track them.
    const int slot = warp - C::kIssuerWarp;
    const uint64_t dK0 = G::kmajor(sbase + C::kOffStages, kTileN, 0);
    const uint64_t dQ0 = G::kmajor(sbase + C::kOffQ, MP, 0);
    const uint64_t dZ0 = G::mnmajor(sbase + C::kOffZ, MP, 0);
    // the low parts (split precision) sit 2 kLatBytes further: one descriptor offset
    constexpr uint32_t kLoStep = static_cast<uint32_t>(2 * C::kLatBytes) >> 4;
    const uint32_t tS = tmem + slot * C::kSlotCols;
    auto wait_stage = [&](int t) -> bool {
      return ptx::mbar_wait(&full[t % NS], (t / NS) & 1, s_abort, args.wait_ns);
    };
    // Q.K^T of tile t over latent half h ([128 h, +128), N = 128), or over
    // all MP latents (h < 0)
    auto issue_qk = [&](int t, int h) {
      const uint64_t dK = dK0 + static_cast<uint32_t>((t % NS) * (C::kTileBytes >> 4));
      const uint64_t dQ = dQ0 + static_cast<uint32_t>(((h > 0 ? h : 0) * kLatRows * G::kRowBytes) >> 4);
      const uint32_t tD = tS + (h > 0 ? h * kLatRows : 0);
      const uint32_t idesc = h < 0 ? C::kIdescQK : C::kIdescQKHalf;
#pragma unroll
      for (int part = 0; part < C::kLatParts; ++part)
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          ptx::mma_ss(tD, dK + G::kmajor_step(kTileN, k), dQ + part * kLoStep + G::kmajor_step(MP, k), idesc,
                      (k > 0 || part > 0) ? 1u : 0u);
    };
    auto commit_s = [&](int t) {
      ptx::mma_commit(&S_full[slot]);
      ptx::mma_commit(&empty[t % NS]);  // both halves of Q.K^T(t) have read the stage
    };
    bool ok = __all_sync(0xffffffffu, ptx::mbar_wait(qz_full, 0, s_abort, args.wait_ns));
    // this slot's tiles: t = slot + 2 i
    if (ok && slot < T) {
      ok = __all_sync(0xffffffffu, wait_stage(slot));
      if (ok) {
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          issue_qk(slot, -1);
          commit_s(slot);
        }
        __syncwarp();
      }
    }
    // Batch of tile t: P(t).V, then the part of Q.K^T(t + 2) whose columns
    // hold no O (MP = 256: latents 128-255; MP = 128: all of S, O lies past
    // it); with MP = 256 the other half follows once O has been read.  With
    // MP = 128 the next P.V waits for O to be read instead.
    for (int i = 0; ok && slot + 2 * i < T; ++i) {
      const int t = slot + 2 * i;
      const bool next = t + 2 < T;
      ok = __all_sync(0xffffffffu, ptx::mbar_wait(&P_full[slot], i & 1, s_abort, args.wait_ns) &&
                                       (MP == 256 || i == 0 ||
                                        ptx::mbar_wait(&O_free[slot], (i - 1) & 1, s_abort, args.wait_ns)) &&
                                       (!next || wait_stage(t + 2)));
      if (!ok) break;
      ptx::tc_fence_after();
      if (ptx::elect_one()) {
#pragma unroll
        for (int part = 0; part < C::kLatParts; ++part)
#pragma unroll
          for (int k = 0; k < MP / 16; ++k)
            ptx::mma_ts(tS + C::kColO, tS + C::col_pk(k), dZ0 + part * kLoStep + G::mnmajor_step(k), C::kIdescPV,
                        (k > 0 || part > 0) ? 1u : 0u);
        ptx::mma_commit(&O_full[slot]);
        if (next) {
          if constexpr (MP == 256) {
            issue_qk(t + 2, 1);
          } else {
            issue_qk(t + 2, -1);
            commit_s(t + 2);
          }
        }
      }
      __syncwarp();
      if (MP == 256 && next) {
        // latents 0-127 share their columns with O: once both groups have read it
        ok = __all_sync(0xffffffffu, ptx::mbar_wait(&O_free[slot], i & 1, s_abort, args.wait_ns));
        if (!ok) break;
        ptx::tc_fence_after();
        if (ptx::elect_one()) {
          issue_qk(t + 2, 0);
          commit_s(t + 2);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) {
      record_error(args.status, kErrTimeout, kSiteDecMma);
      *s_abort = 1;
    }
    // Drain: every lane commits (a lane that issued nothing arrives at once).
    ptx::mma_commit(drain);
    ptx::mbar_wait_drain(drain, 0);
  } else {
    // ------------------------------------------------------------ softmax / epilogue groups
    const int s = warp >> 3;  // slot
    float zscale = 1.f;
    if constexpr (PREC != 0) {
      zscale = stage_z_f16<D, MP, NS, PREC>(args, smem, threadIdx.x);
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(qz_full);
    }
    DecodeGroup<D, MP, NS, PREC> grp{args, tmem, warp, lane, s, tile0, T, S_full, P_full, O_full, O_free, turn,
                               s_xm + (s * 2) * 128, s_xl + (s * 2) * 128, s_abort, zscale};
    if ((warp >> 2) & 1) grp.template run<1>(); else grp.template run<0>();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kProducerWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace flare
