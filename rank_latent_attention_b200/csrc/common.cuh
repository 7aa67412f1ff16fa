// Shared definitions of the FLARE++ kernels: status codes, the device status
// word, tile geometry of the bf16 tensor-core path and smem descriptor helpers.
#pragma once

#include <stdint.h>

#include "ptx_sm100.cuh"

namespace flare {

// Status codes shared with include/flarepp.h.
enum : int {
  kOk = 0,
  kErrInvalidArg = 1,
  kErrUnsupported = 2,
  kErrCuda = 3,
  kErrTimeout = 4,
};

// Where a bounded wait gave up (second word of the device status).
enum : int {
  kSiteEncProducer = 1,
  kSiteEncMma = 2,
  kSiteEncSoftmax = 3,
  kSiteDecProducer = 4,
  kSiteDecMma = 5,
  kSiteDecSoftmax = 6,
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTileN = 128;   // tokens per tile (MMA M of the decode, N of the encode)
constexpr int kLatRows = 128; // latent rows per tcgen05 MMA (M = 128, cta_group::1)

// 2^x on the FMA/ALU pipes, for the share of a softmax tile's exponentials
// that would otherwise queue behind the MUFU unit (16 results per clock per
// SM on sm_100, the binding resource of the softmax).  For -125 <= x <= 64 the
// relative error is below 7.5e-5 (P is then rounded to bf16, 2^-9); x < -125
// gives about 2^-125 (2.4e-38) in place of a smaller value.  The clamp keeps
// the exponent field of the result at 1 or more: p(f) can fall just below 1,
// and 2^-126 scaling would then produce a denormal.
//   x = j + f with j = rint(x), f in [-1/2, 1/2]: adding 1.5 * 2^23 leaves j
//   in the low mantissa bits of the sum, and subtracting it back gives j
//   exactly; 2^f is the degree-3 polynomial of minimax relative error on
//   [-1/2, 1/2] (Remez exchange, coefficients printed by exp2_poly_fit.py);
//   2^j scales it by adding j to the exponent field (the sum's bits shifted
//   left by 23 are j << 23, the constant's bits shift out).
__device__ __forceinline__ float exp2_poly3(float x) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  const float xc = fmaxf(x, -125.f);
  const float r = __fadd_rn(xc, kRound);
  const float f = __fadd_rn(xc, -__fadd_rn(r, -kRound));
  float p = fmaf(0.0551716685f, f, 0.242611125f);
  p = fmaf(p, f, 0.693260968f);
  p = fmaf(p, f, 0.999928057f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(r) << 23));
}

// exp2_poly3 on a packed pair (lo, hi): the same steps, the fp32 adds and
// multiply-adds as f32x2 instructions.
__device__ __forceinline__ uint64_t exp2_poly3_x2(uint64_t x) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  float x0, x1;
  ptx::f2_split(x, x0, x1);
  const uint64_t xc = ptx::f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t r = ptx::add2(xc, ptx::f2(kRound, kRound));
  const uint64_t j = ptx::add2(r, ptx::f2(-kRound, -kRound));
  const uint64_t f = ptx::fma2(j, ptx::f2(-1.f, -1.f), xc);  // xc - j, exact product, one rounding
  uint64_t p = ptx::fma2(ptx::f2(0.0551716685f, 0.0551716685f), f, ptx::f2(0.242611125f, 0.242611125f));
  p = ptx::fma2(p, f, ptx::f2(0.693260968f, 0.693260968f));
  p = ptx::fma2(p, f, ptx::f2(0.999928057f, 0.999928057f));
  float p0, p1, r0, r1;
  ptx::f2_split(p, p0, p1);
  ptx::f2_split(r, r0, r1);
  return ptx::f2(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(r0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(r1) << 23)));
}

// Record the first failure in the device status word {code, site}.
__device__ __forceinline__ void record_error(int* status, int code, int site) {
  if (atomicCAS(status, 0, code) == 0) atomicExch(status + 1, site);
}

// Geometry of a [rows][D] bf16 tile in shared memory as written by a TMA
// load with the swizzle matching its row width:
//   D <= 64 : one block, row pitch 2*D bytes (32/64/128 B swizzle);
//   D == 128: two 64-column blocks of [rows][64], each with 128 B rows.
template <int D>
struct TileGeom {
  static_assert(D == 16 || D == 32 || D == 64 || D == 128, "D must be 16, 32, 64 or 128");
  static constexpr int kRowBytes = D >= 64 ? 128 : 2 * D;   // row pitch inside one column block
  static constexpr int kBlocks = D > 64 ? D / 64 : 1;        // 64-column blocks
  static constexpr int kBoxCols = D >= 64 ? 64 : D;          // TMA box inner extent (elements)
  static constexpr uint32_t kSwizzle = D >= 64 ? 2u : (D == 32 ? 4u : 6u);  // descriptor code
  static constexpr int kAtomBytes = 8 * kRowBytes;           // 8-row swizzle atom

  // K-major operand (rows = M or N of the MMA, D = reduction dim), K step k of 16.
  __device__ static __forceinline__ uint64_t kmajor(uint32_t base, int rows, int k) {
    // 16 elements = 32 bytes along the row; past 64 elements, the next column block.
    const int elem = k * 16;
    const uint32_t addr = base + (elem / 64) * rows * 128 + (elem % 64) * 2;
    return ptx::smem_desc(addr, 16, kAtomBytes, kSwizzle);
  }
  // MN-major operand (rows = reduction dim, D = N of the MMA), K step k of 16 rows.
  __device__ static __forceinline__ uint64_t mnmajor(uint32_t base, int rows, int k) {
    const uint32_t addr = base + k * 16 * kRowBytes;
    return ptx::smem_desc(addr, rows * 128, kAtomBytes, kSwizzle);
  }
  static constexpr int bytes(int rows) { return rows * D * 2; }

  // The same descriptors as base + offset: only the start-address field
  // (bits [0,14), 16-byte units) moves between K steps and ring stages, so
  // the MMA issuer adds a constant instead of rebuilding 64-bit descriptors.
  __host__ __device__ static constexpr uint32_t kmajor_step(int rows, int k) {
    return static_cast<uint32_t>(((k * 16) / 64) * rows * 128 + ((k * 16) % 64) * 2) >> 4;
  }
  __host__ __device__ static constexpr uint32_t mnmajor_step(int k) {
    return static_cast<uint32_t>(k * 16 * kRowBytes) >> 4;
  }
};

}  // namespace flare
