// C ABI of the FLARE++ mixer forward (include/flarepp.h): argument checks,
// workspace layout, TMA descriptors and kernel dispatch.  Every step of the
// computation runs in the kernels included below; this file only marshals.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>

#include <algorithm>
#include <limits>
#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include <type_traits>

#include "../../include/flarepp.h"
#include "backward_simt.cuh"
#include "backward_tc.cuh"
#include "comm_tc.cuh"
#include "decode_tc.cuh"
#include "encode_tc.cuh"
#include "merge.cuh"
#include "simt_f32.cuh"

namespace flare {
namespace {

__device__ int g_status[2];  // {first error code, site} per device

std::atomic<int> g_split_override{0};
// Programmatic dependent launch of a mixer call's later kernels: -1 by size
// (overlap_launches), 0 never, 1 always (flare_set_launch_overlap)
std::atomic<int> g_launch_overlap{-1};
std::atomic<int> g_wait_ms{2000};
thread_local int t_last_launches = 0;
// The split override as this thread's current entry-point call first read
// it (-1 outside a call): every split count inside one call, the workspace
// check's and the kernels' alike, comes from the same value even if another
// thread changes the override meanwhile.
thread_local int t_split_pin = -1;

struct SplitPin {
  int prev;
  SplitPin() : prev(t_split_pin) {
    if (prev < 0) t_split_pin = g_split_override.load();
  }
  ~SplitPin() { t_split_pin = prev; }
};

constexpr int kMaxDevices = 64;

// ------------------------------------------------------------------ launch profiling
// When enabled (flare_profile_begin), every kernel launch is bracketed by two
// CUDA events on the launching stream; flare_profile_end returns the
// durations.  Events only, no synchronisation until the end.
struct Profile {
  std::mutex mu;
  bool on = false;
  int cap = 0, used = 0;
  std::vector<cudaEvent_t> ev;
  std::vector<int> kind;
};
Profile g_prof;

struct ProfScope {
  int slot = -1;
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t s) : st(s) {
    std::lock_guard<std::mutex> lock(g_prof.mu);
    if (!g_prof.on || g_prof.used >= g_prof.cap) return;
    slot = g_prof.used++;
    g_prof.kind[slot] = kind;
    cudaEventRecord(g_prof.ev[2 * slot], st);
  }
  ~ProfScope() {
    if (slot >= 0) cudaEventRecord(g_prof.ev[2 * slot + 1], st);
  }
};

int* status_ptr() {
  static int* ptrs[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) {
      cudaGetLastError();  // the failed lookup must not read as a later launch's error
      return nullptr;
    }
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int check_sizes(int B, int H, int64_t N, int M, int D, int dtype) {
  if (dtype != FLARE_F32 && dtype != FLARE_BF16 && dtype != FLARE_BF16_F32OUT) return FLARE_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || M < 1) return FLARE_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H > 65535) return FLARE_ERR_UNSUPPORTED;
  if (N >= (int64_t(1) << 31) - 256) return FLARE_ERR_UNSUPPORTED;
  if (!(D == 16 || D == 32 || D == 64 || D == 128)) return FLARE_ERR_UNSUPPORTED;
  if (M > 256) return FLARE_ERR_UNSUPPORTED;
  if (dtype == FLARE_BF16 && M % 16 != 0) return FLARE_ERR_UNSUPPORTED;
  return FLARE_OK;
}

bool device_ptr(const void* p) {
  if (!p || (reinterpret_cast<uintptr_t>(p) & 15u)) return false;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

// CTAs per head along the token axis.  A kernel's time is about
//   (waves of the SMs' CTA slots) x (tiles per CTA + a fixed cost per CTA),
// waves = ceil(BH s / slots) with per_sm resident CTAs per SM; the fixed
// cost (launch share, barrier and TMEM set-up, the first loads, the
// epilogue: about 384 tokens' worth of work) makes fewer, longer CTAs win
// ties.  The count minimising that estimate is taken among s from the
// smallest that keeps a CTA at most ~32768 tokens, over eight more waves'
// worth of CTAs per head.  Rounding the split count up to fill the waves
// instead sent few-head workloads just past a wave boundary (32 heads: 5
// splits, 160 CTAs = 1.08 waves, twice the time of 4 splits).
// `tile` is the kernel's token tile (64 for the encode, 128 for the decode).
int choose_splits(int BH, int64_t N, int tile, int per_sm = 1) {
  const int64_t tiles = ceil_div(N, tile);
  int64_t s = t_split_pin >= 0 ? t_split_pin : g_split_override.load();
  if (s <= 0) {
    const int64_t slots = int64_t(sm_count()) * per_sm;
    const int64_t fixed_tiles = std::max<int64_t>(1, 384 / tile);
    const int64_t lo = std::max<int64_t>(1, ceil_div(tiles, 32768 / tile));
    const int64_t hi = std::min<int64_t>(tiles, lo + 8 * ceil_div(slots, BH));
    int64_t best = std::numeric_limits<int64_t>::max();
    for (int64_t c = lo; c <= hi; ++c) {
      const int64_t cost = ceil_div(int64_t(BH) * c, slots) * (ceil_div(tiles, c) + fixed_tiles);
      if (cost < best) {
        best = cost;
        s = c;
      }
    }
  }
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(s, tiles)));
}

// Partials per head produced by one encode: one per split on the CUDA-core
// path; on the tensor-core path one per (split, slot, buffer) accumulator.
int partials(int M, int D, int splits, int dtype) {
  if (dtype != FLARE_BF16) return splits;
  return splits * encode_partials_per_split(D, M > kLatRows ? 2 : 1);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct EncodeWs {
  float* O;
  float* m;
  float* l;
  size_t bytes;
};

EncodeWs encode_ws_layout(char* base, int BH, int64_t N, int M, int D, int dtype) {
  const int P = partials(M, D, choose_splits(BH, N, kEncTile), dtype);
  const size_t rows = static_cast<size_t>(BH) * P * M;
  EncodeWs w;
  size_t off = 0;
  w.O = reinterpret_cast<float*>(base + off);
  off += align256(rows * D * sizeof(float));
  w.m = reinterpret_cast<float*>(base + off);
  off += align256(rows * sizeof(float));
  w.l = reinterpret_cast<float*>(base + off);
  off += align256(rows * sizeof(float));
  w.bytes = off;
  return w;
}

// Storage size of Q_dyn / Z (and of Y): bf16 only on the tensor-core path.
size_t elem_size(int dtype) { return dtype == FLARE_BF16 ? 2 : 4; }

// ------------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 3-D bf16 map over [planes][rows][D] with a {min(D,64), box_rows, 1} box and
// the swizzle that matches the tile geometry the kernels expect.
bool make_map(CUtensorMap* map, const void* ptr, int D, int64_t rows, int64_t planes, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(planes)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows) * D * 2};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(D >= 64 ? 64 : D), static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = D >= 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                        : (D == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launchers
// Launch with programmatic stream serialisation when pdl is set: the kernel
// may start while the previous kernel of the stream finishes.  Only kernels
// that wait (grid_dep_wait) before reading anything an earlier kernel of the
// call writes are launched that way: the merges, and the routing encode and
// the decode of a mixer call, whose K and V are the call's inputs.
template <typename... Exp, typename... Act>
cudaError_t launch_k(bool pdl, void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Act&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

// Encode tiles per CTA up to which a mixer call overlaps launches by default.
constexpr int64_t kOverlapMaxTilesPerCta = 64;

// Whether a mixer call overlaps its kernels' prologues with the kernels
// before them.  By default only when each encode CTA has few tiles: there the
// fixed cost of a kernel (launch, barrier and TMEM set-up, the first loads)
// is a large share of the call; on long token runs the overlap was measured
// slower (the early CTAs' Q load waits behind their K/V prefetch).
bool overlap_launches(int BH, int64_t N) {
  const int mode = g_launch_overlap.load();
  if (mode >= 0) return mode > 0;
  const int64_t tiles = ceil_div(N, kEncTile);
  return ceil_div(tiles, choose_splits(BH, N, kEncTile)) <= kOverlapMaxTilesPerCta;
}

// Tensor maps of one encode: Q (hi), K, V, and the low parts of Q (split
// precision; a copy of Q's map otherwise, never read).
struct EncodeMaps {
  CUtensorMap q, k, v, qlo;
};

template <int D, int NHALF, int NS, int PREC>
cudaError_t launch_encode_tc_t(const EncodeMaps& m, const EncodeArgs& a, int BH, cudaStream_t st, bool pdl) {
  using C = EncodeCfg<D, NHALF, NS, PREC>;
  auto kern = encode_tc_kernel<D, NHALF, NS, PREC>;
  static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  return launch_k(pdl, kern, dim3(a.splits, BH), dim3(C::kThreads), C::kSmemBytes, st, m.q, m.k, m.v, m.qlo, a);
}

template <int NHALF, int PREC>
cudaError_t launch_encode_tc_n(int D, const EncodeMaps& m, const EncodeArgs& a, int BH, cudaStream_t st, bool pdl) {
  switch (D) {
    case 16: return launch_encode_tc_t<16, NHALF, 16, PREC>(m, a, BH, st, pdl);
    case 32: return launch_encode_tc_t<32, NHALF, 8, PREC>(m, a, BH, st, pdl);
    case 64: return launch_encode_tc_t<64, NHALF, 8, PREC>(m, a, BH, st, pdl);
    default:
      if constexpr (PREC == 0) return launch_encode_tc_t<128, NHALF, NHALF == 2 ? 4 : 5, 0>(m, a, BH, st, pdl);
      return cudaErrorInvalidValue;  // split precision: D <= 64 only (checked by the caller)
  }
}

cudaError_t launch_encode_tc(int D, int M, int prec, const EncodeMaps& m, const EncodeArgs& a, int BH,
                             cudaStream_t st, bool pdl) {
  if (M > kLatRows) {
    if (prec == 2) return launch_encode_tc_n<2, 2>(D, m, a, BH, st, pdl);
    if (prec == 1) return launch_encode_tc_n<2, 1>(D, m, a, BH, st, pdl);
    return launch_encode_tc_n<2, 0>(D, m, a, BH, st, pdl);
  }
  if (prec == 2) return launch_encode_tc_n<1, 2>(D, m, a, BH, st, pdl);
  if (prec == 1) return launch_encode_tc_n<1, 1>(D, m, a, BH, st, pdl);
  return launch_encode_tc_n<1, 0>(D, m, a, BH, st, pdl);
}

// Tensor maps of one decode: K, Q (hi), Z, and the low parts of Q (split
// precision, which reads Z as fp32 instead of through a map; unused maps are
// copies of Q's, never read).
struct DecodeMaps {
  CUtensorMap k, q, z, qlo, zlo;
};

template <int D, int MP, int NS, int PREC>
cudaError_t launch_decode_tc_t(const DecodeMaps& m, const DecodeArgs& a, int BH, cudaStream_t st, bool pdl) {
  using C = DecodeCfg<D, MP, NS, PREC>;
  auto kern = decode_tc_kernel<D, MP, NS, PREC>;
  static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  return launch_k(pdl, kern, dim3(a.splits, BH), dim3(C::kThreads), C::kSmemBytes, st, m.k, m.q, m.z, m.qlo, m.zlo,
                  a);
}

template <int MP, int PREC>
cudaError_t launch_decode_tc_m(int D, const DecodeMaps& m, const DecodeArgs& a, int BH, cudaStream_t st, bool pdl) {
  switch (D) {
    case 16: return launch_decode_tc_t<16, MP, 8, PREC>(m, a, BH, st, pdl);
    case 32: return launch_decode_tc_t<32, MP, 8, PREC>(m, a, BH, st, pdl);
    // split precision holds four resident latent blocks: a shallower K ring
    case 64: return launch_decode_tc_t<64, MP, (PREC && MP == 256) ? 5 : 8, PREC>(m, a, BH, st, pdl);
    default:
      if constexpr (PREC == 0) return launch_decode_tc_t<128, MP, 2, 0>(m, a, BH, st, pdl);
      return cudaErrorInvalidValue;  // split precision: D <= 64 only (checked by the caller)
  }
}

template <int D, typename TQ, typename TKV>
cudaError_t launch_encode_f32_t(const EncodeF32Args& a, int BH, cudaStream_t st) {
  constexpr int RPB = 256 / (D / (D < 32 ? D : 32));
  encode_f32_kernel<D, TQ, TKV><<<dim3(a.splits, BH, static_cast<unsigned>(ceil_div(a.M, RPB))), 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename TQ, typename TKV>
cudaError_t launch_encode_f32_d(int D, const EncodeF32Args& a, int BH, cudaStream_t st) {
  switch (D) {
    case 16: return launch_encode_f32_t<16, TQ, TKV>(a, BH, st);
    case 32: return launch_encode_f32_t<32, TQ, TKV>(a, BH, st);
    case 64: return launch_encode_f32_t<64, TQ, TKV>(a, BH, st);
    default: return launch_encode_f32_t<128, TQ, TKV>(a, BH, st);
  }
}

template <int D, typename TK>
cudaError_t launch_decode_f32_t(const DecodeF32Args& a, int BH, cudaStream_t st) {
  decode_f32_kernel<D, TK><<<dim3(static_cast<unsigned>(ceil_div(a.N, 8)), BH), 256, 0, st>>>(a);
  return cudaGetLastError();
}

template <typename TK>
cudaError_t launch_decode_f32_d(int D, const DecodeF32Args& a, int BH, cudaStream_t st) {
  switch (D) {
    case 16: return launch_decode_f32_t<16, TK>(a, BH, st);
    case 32: return launch_decode_f32_t<32, TK>(a, BH, st);
    case 64: return launch_decode_f32_t<64, TK>(a, BH, st);
    default: return launch_decode_f32_t<128, TK>(a, BH, st);
  }
}

// Merge of one encode's split partials ([BH][P][M] in the workspace) into
// `out`; lse_out (optional) receives the natural-log log-sum-exp per latent.
template <typename T>
cudaError_t launch_merge(const EncodeWs& w, void* out, float* lse_out, int BH, int P, int M, int D,
                         cudaStream_t st, bool pdl, SplitOut split = SplitOut{nullptr, nullptr}) {
  const MergeGeom g{P, M, D, static_cast<long long>(P) * M * D, static_cast<long long>(M) * D,
                    static_cast<long long>(P) * M, M};
  return launch_k(pdl, lse_merge_kernel<T, false>, dim3(static_cast<unsigned>(ceil_div(int64_t(M) * D, 256)), BH),
                  dim3(256), 0, st, static_cast<const float*>(w.O), static_cast<const float*>(w.m),
                  static_cast<const float*>(w.l), static_cast<T*>(out), lse_out, g, split);
}

// The split-precision tensor-core form of FLARE_BF16_F32OUT covers M % 16 == 0
// and D <= 64; other sizes of that mode run on the CUDA-core kernels.
bool f32out_on_tensor_cores(int M, int D) { return M % 16 == 0 && D <= 64; }

// ------------------------------------------------------------------ steps
// One encode (partials + merge) into `out`; Q indexed per q_batched.
// dtype FLARE_BF16: everything bf16, tensor cores.  FLARE_F32: everything
// fp32.  FLARE_BF16_F32OUT: K, V bf16, out fp32, Q bf16 if q_bf16 else fp32
// (CUDA cores), or with prec > 0 the split-precision tensor-core encode:
// prec 1 takes bf16 Q, prec 2 takes Q as bf16 parts Q (hi) and Q_lo; `split`
// (optional) also receives the fp32 result as a hi/lo bf16 pair.
// lse_out: when set, `out` is fp32 whatever the dtype and the merge also
// writes the natural-log log-sum-exp of each latent's logits ([B][H][M]).
int run_encode(const void* Q, int q_batched, const void* K, const void* V, void* out, int B, int H, int64_t N,
               int M, int D, int dtype, char* ws, cudaStream_t st, int* launches, bool q_bf16 = false,
               float* lse_out = nullptr, bool f32_out = false, int prec = 0, const void* Q_lo = nullptr,
               SplitOut split = SplitOut{nullptr, nullptr}, bool pdl = false, bool pdl_merge = false) {
  const int BH = B * H;
  const int splits = choose_splits(BH, N, kEncTile);
  const int P = partials(M, D, splits, dtype);
  const EncodeWs w = encode_ws_layout(ws, BH, N, M, D, dtype);
  int* status = status_ptr();
  if (!status) return FLARE_ERR_CUDA;
  cudaError_t e;
  if (dtype == FLARE_BF16 || prec > 0) {
    EncodeMaps maps;
    if (!make_map(&maps.q, Q, D, M, q_batched ? BH : H, kLatRows) || !make_map(&maps.k, K, D, N, BH, kEncTile) ||
        !make_map(&maps.v, V, D, N, BH, kEncTile))
      return FLARE_ERR_CUDA;
    if (prec == 2) {
      if (!make_map(&maps.qlo, Q_lo, D, M, q_batched ? BH : H, kLatRows)) return FLARE_ERR_CUDA;
    } else {
      maps.qlo = maps.q;
    }
    EncodeArgs a;
    a.Q = Q;
    a.Q_lo = prec == 2 ? Q_lo : Q;
    a.N = static_cast<int>(N);
    a.M = M;
    a.q_batched = q_batched;
    a.H = H;
    a.splits = splits;
    a.tiles = static_cast<int>(ceil_div(N, kEncTile));
    a.P = P;
    a.O_part = w.O;
    a.m_part = w.m;
    a.l_part = w.l;
    a.status = status;
    a.wait_ns = static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull;
    // one split per head: the encode writes the result itself, no merge
    a.direct = P == 1 ? 1 : 0;
    a.out = out;
    a.out_f32 = (f32_out || prec > 0) ? 1 : 0;
    a.lse_out = lse_out;
    a.out_hi = split.hi;
    a.out_lo = split.lo;
    {
      ProfScope prof(FLARE_KERNEL_ENCODE_TC, st);
      e = launch_encode_tc(D, M, prec, maps, a, BH, st, pdl);
    }
    if (e != cudaSuccess) return FLARE_ERR_CUDA;
    if (a.direct) {
      *launches += 1;
      return FLARE_OK;
    }
    ProfScope prof(FLARE_KERNEL_MERGE, st);
    e = (f32_out || prec > 0) ? launch_merge<float>(w, out, lse_out, BH, P, M, D, st, pdl_merge, split)
                              : launch_merge<__nv_bfloat16>(w, out, lse_out, BH, P, M, D, st, pdl_merge);
  } else {
    EncodeF32Args a;
    a.N = static_cast<int>(N);
    a.M = M;
    a.q_batched = q_batched;
    a.H = H;
    a.splits = splits;
    a.tiles = static_cast<int>(ceil_div(N, kTileN));
    a.P = P;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.O_part = w.O;
    a.m_part = w.m;
    a.l_part = w.l;
    {
      ProfScope prof(FLARE_KERNEL_ENCODE_F32, st);
      if (dtype == FLARE_F32)
        e = launch_encode_f32_d<float, float>(D, a, BH, st);
      else if (q_bf16)
        e = launch_encode_f32_d<__nv_bfloat16, __nv_bfloat16>(D, a, BH, st);
      else
        e = launch_encode_f32_d<float, __nv_bfloat16>(D, a, BH, st);
    }
    if (e != cudaSuccess) return FLARE_ERR_CUDA;
    ProfScope prof(FLARE_KERNEL_MERGE, st);
    e = launch_merge<float>(w, out, lse_out, BH, P, M, D, st, false);
  }
  *launches += 2;
  return e == cudaSuccess ? FLARE_OK : FLARE_ERR_CUDA;
}

// One decode into Y.  With `lo` (FLARE_BF16_F32OUT on the tensor cores), Q
// is the hi part of the bf16 pair whose low part is lo->Q_lo, Z is read as
// fp32 from lo->Zf (the `Z` argument is unused), and Y is fp32.
struct DecodeLo {
  const void* Q_lo;
  const float* Zf;
};

int run_decode(const void* K, const void* Q, int q_batched, const void* Z, void* Y, int B, int H, int64_t N, int M,
               int D, int dtype, cudaStream_t st, int* launches, const DecodeLo* lo = nullptr, bool pdl = false) {
  const int BH = B * H;
  cudaError_t e;
  if (dtype == FLARE_BF16 || lo) {
    int* status = status_ptr();
    if (!status) return FLARE_ERR_CUDA;
    DecodeMaps maps;
    if (!make_map(&maps.k, K, D, N, BH, kTileN) || !make_map(&maps.q, Q, D, M, q_batched ? BH : H, kLatRows))
      return FLARE_ERR_CUDA;
    if (lo) {
      if (!make_map(&maps.qlo, lo->Q_lo, D, M, q_batched ? BH : H, kLatRows)) return FLARE_ERR_CUDA;
      maps.z = maps.q;
    } else {
      if (!make_map(&maps.z, Z, D, M, BH, kLatRows)) return FLARE_ERR_CUDA;
      maps.qlo = maps.q;
    }
    maps.zlo = maps.q;
    DecodeArgs a;
    a.N = static_cast<int>(N);
    a.M = M;
    a.q_batched = q_batched;
    a.H = H;
    a.splits = choose_splits(BH, N, kTileN);
    a.tiles = static_cast<int>(ceil_div(N, kTileN));
    a.Y = Y;
    a.Zf = lo ? lo->Zf : nullptr;
    a.status = status;
    a.wait_ns = static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull;
    ProfScope prof(FLARE_KERNEL_DECODE_TC, st);
    if (lo)
      e = M > kLatRows ? launch_decode_tc_m<256, 1>(D, maps, a, BH, st, pdl)
                       : launch_decode_tc_m<128, 1>(D, maps, a, BH, st, pdl);
    else
      e = M > kLatRows ? launch_decode_tc_m<256, 0>(D, maps, a, BH, st, pdl)
                       : launch_decode_tc_m<128, 0>(D, maps, a, BH, st, pdl);
  } else {
    DecodeF32Args a;
    a.N = static_cast<int>(N);
    a.M = M;
    a.q_batched = q_batched;
    a.H = H;
    a.K = K;
    a.Q = static_cast<const float*>(Q);
    a.Z = static_cast<const float*>(Z);
    a.Y = static_cast<float*>(Y);
    ProfScope prof(FLARE_KERNEL_DECODE_F32, st);
    e = dtype == FLARE_F32 ? launch_decode_f32_d<float>(D, a, BH, st) : launch_decode_f32_d<__nv_bfloat16>(D, a, BH, st);
  }
  *launches += 1;
  return e == cudaSuccess ? FLARE_OK : FLARE_ERR_CUDA;
}

// Workspace of the mixer: the encode's partials, Q_dyn and Z (dtype storage),
// and for FLARE_BF16_F32OUT on the tensor cores the hi and lo bf16 parts of
// Q_dyn.
size_t mix_split_part_bytes(int BH, int M, int D, int dtype) {
  if (dtype != FLARE_BF16_F32OUT || !f32out_on_tensor_cores(M, D)) return 0;
  return align256(static_cast<size_t>(BH) * M * D * 2);
}

size_t mix_ws_bytes(int B, int H, int64_t N, int M, int D, int dtype) {
  const int BH = B * H;
  const size_t enc = encode_ws_layout(nullptr, BH, N, M, D, dtype).bytes;
  const size_t lat = align256(static_cast<size_t>(BH) * M * D * elem_size(dtype));
  return enc + 2 * lat + 2 * mix_split_part_bytes(BH, M, D, dtype);
}

// Scratch resolution: caller's buffer, or a stream-ordered allocation.
struct Scratch {
  char* ptr = nullptr;
  bool owned = false;
};

int get_scratch(void* ws, size_t have, size_t need, cudaStream_t st, Scratch* out) {
  if (ws) {
    if (have < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return FLARE_ERR_INVALID_ARG;
    out->ptr = static_cast<char*>(ws);
    return FLARE_OK;
  }
  void* p = nullptr;
  if (cudaMallocAsync(&p, need, st) != cudaSuccess) return FLARE_ERR_CUDA;
  out->ptr = static_cast<char*>(p);
  out->owned = true;
  return FLARE_OK;
}

int release_scratch(const Scratch& s, cudaStream_t st) {
  if (s.owned && cudaFreeAsync(s.ptr, st) != cudaSuccess) return FLARE_ERR_CUDA;
  return FLARE_OK;
}

int mix_impl(const void* seeds, const void* K, const void* V, void* Y, void* Qd_out, void* Z_out, int B, int H,
             int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream,
             float* lse1_out = nullptr, float* lse2_out = nullptr) {
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (!device_ptr(seeds) || !device_ptr(K) || !device_ptr(V) || !device_ptr(Y)) return FLARE_ERR_INVALID_ARG;
  if ((Qd_out || Z_out) && (!device_ptr(Qd_out) || !device_ptr(Z_out))) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes, mix_ws_bytes(B, H, N, M, D, dtype), st, &s);
  if (rc) return rc;
  const size_t enc = encode_ws_layout(nullptr, BH, N, M, D, dtype).bytes;
  const size_t lat = align256(static_cast<size_t>(BH) * M * D * elem_size(dtype));
  void* Qd = Qd_out ? Qd_out : s.ptr + enc;
  void* Z = Z_out ? Z_out : s.ptr + enc + lat;
  int launches = 0;
  // the merges, the routing encode and the decode may start while the kernel
  // before each finishes (K and V are the call's inputs, not that kernel's
  // output)
  const bool pdl = overlap_launches(BH, N);
  if (const size_t pb = mix_split_part_bytes(BH, M, D, dtype)) {
    // FLARE_BF16_F32OUT on the tensor cores: the seed encode's merge also
    // writes Q_dyn as hi/lo bf16 parts, the query operands of the routing
    // encode and the key operands of the decode; the decode reads the fp32 Z
    // and makes its own fp16 parts
    char* parts = s.ptr + enc + 2 * lat;
    auto* Qhi = reinterpret_cast<__nv_bfloat16*>(parts);
    auto* Qlo = reinterpret_cast<__nv_bfloat16*>(parts + pb);
    rc = run_encode(seeds, 0, K, V, Qd, B, H, N, M, D, dtype, s.ptr, st, &launches, true, lse1_out, false, 1,
                    nullptr, SplitOut{Qhi, Qlo}, false, pdl);
    if (!rc)
      rc = run_encode(Qhi, 1, K, V, Z, B, H, N, M, D, dtype, s.ptr, st, &launches, false, lse2_out, false, 2, Qlo,
                      SplitOut{nullptr, nullptr}, pdl, pdl);
    const DecodeLo lo{Qlo, static_cast<const float*>(Z)};
    if (!rc) rc = run_decode(K, Qhi, 1, nullptr, Y, B, H, N, M, D, dtype, st, &launches, &lo, pdl);
  } else {
    // the seed encode waits for whatever came before the call (it may write K/V)
    rc = run_encode(seeds, 0, K, V, Qd, B, H, N, M, D, dtype, s.ptr, st, &launches, /*q_bf16=*/true, lse1_out,
                    false, 0, nullptr, SplitOut{nullptr, nullptr}, false, pdl);
    if (!rc)
      rc = run_encode(Qd, 1, K, V, Z, B, H, N, M, D, dtype, s.ptr, st, &launches, false, lse2_out, false, 0, nullptr,
                      SplitOut{nullptr, nullptr}, pdl, pdl);
    if (!rc) rc = run_decode(K, Qd, 1, Z, Y, B, H, N, M, D, dtype, st, &launches, nullptr, pdl);
  }
  const int rc2 = release_scratch(s, st);
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

}  // namespace
}  // namespace flare

using namespace flare;

// ------------------------------------------------------------------ communication matrix
// C = W_enc W_dec (M x M per head) from the existing steps: a decode with
// Z = columns [j D, j D + D) of the M x M identity gives those columns of
// W_dec = softmax_M(K Q^T) (N x M), and an encode with that block as V gives
// the same columns of C = softmax_N(Q K^T) W_dec.
template <typename T>
__device__ __forceinline__ T from_float(float v);
template <>
__device__ __forceinline__ float from_float<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Zid[bh][m][d] = 1 if m == j D + d, else 0.
template <typename T>
__global__ void identity_block_kernel(T* Z, size_t total, int M, int D, int j) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int d = static_cast<int>(idx % D);
  const int m = static_cast<int>((idx / D) % M);
  Z[idx] = from_float<T>(m == j * D + d ? 1.f : 0.f);
}

// C[bh][m][j D + d] = Cb[bh][m][d] for the columns inside [0, M).
template <typename T>
__global__ void scatter_block_kernel(const T* Cb, T* C, size_t total, int M, int D, int j) {
  const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int d = static_cast<int>(idx % D);
  const size_t row = idx / D;  // bh * M + m
  const int col = j * D + d;
  if (col < M) C[row * M + col] = Cb[idx];
}

struct CommWs {
  size_t enc, zid, y, cb, bytes;
};

CommWs comm_ws_layout(int B, int H, int64_t N, int M, int D, int dtype) {
  const int BH = B * H;
  const size_t es = elem_size(dtype);
  CommWs w;
  w.enc = encode_ws_layout(nullptr, BH, N, M, D, dtype).bytes;
  w.zid = align256(static_cast<size_t>(BH) * M * D * es);
  w.y = align256(static_cast<size_t>(BH) * N * D * es);
  w.cb = align256(static_cast<size_t>(BH) * M * D * es);
  w.bytes = w.enc + w.zid + w.y + w.cb;
  return w;
}

template <typename T>
int run_comm(const void* Q, int q_batched, const void* K, void* C, int B, int H, int64_t N, int M, int D, int dtype,
             char* ws, cudaStream_t st, int* launches) {
  const int BH = B * H;
  const CommWs w = comm_ws_layout(B, H, N, M, D, dtype);
  T* Zid = reinterpret_cast<T*>(ws + w.enc);
  T* Yj = reinterpret_cast<T*>(ws + w.enc + w.zid);
  T* Cb = reinterpret_cast<T*>(ws + w.enc + w.zid + w.y);
  const size_t blk = static_cast<size_t>(BH) * M * D;
  const unsigned grid = static_cast<unsigned>((blk + 255) / 256);
  for (int j = 0; j * D < M; ++j) {
    identity_block_kernel<T><<<grid, 256, 0, st>>>(Zid, blk, M, D, j);
    if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_CUDA;
    ++*launches;
    int rc = run_decode(K, Q, q_batched, Zid, Yj, B, H, N, M, D, dtype, st, launches);
    if (!rc) rc = run_encode(Q, q_batched, K, Yj, Cb, B, H, N, M, D, dtype, ws, st, launches);
    if (rc) return rc;
    scatter_block_kernel<T><<<grid, 256, 0, st>>>(Cb, static_cast<T*>(C), blk, M, D, j);
    if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_CUDA;
    ++*launches;
  }
  return FLARE_OK;
}

// One pass on the tensor cores (comm_tc.cuh), bf16 inputs: an encode of Q
// over the tokens (K as its values, only its merge's log-sum-exp per latent
// is kept), the C kernel per (token split, latent half, head), and the sum of
// its split partials into C (bf16 or fp32).  Workspace, in order: the
// encode's partials, its [BH][M][D] fp32 output (unused), lse2 [BH][M], the
// C partials [BH][S][M][M] fp32.
struct CommTcWs {
  size_t enc, z, lse, part, bytes;
  int splits;
};

int comm_splits(int BH, int64_t N, int M) {
  // whole waves of the SMs, over the (head, latent half) CTA columns
  return choose_splits(BH * (M > kLatRows ? 2 : 1), N, kTileN);
}

CommTcWs comm_tc_ws_layout(int B, int H, int64_t N, int M, int D) {
  const int BH = B * H;
  CommTcWs w;
  w.splits = comm_splits(BH, N, M);
  w.enc = encode_ws_layout(nullptr, BH, N, M, D, FLARE_BF16).bytes;
  w.z = align256(static_cast<size_t>(BH) * M * D * sizeof(float));
  w.lse = align256(static_cast<size_t>(BH) * M * sizeof(float));
  w.part = align256(static_cast<size_t>(BH) * w.splits * M * M * sizeof(float));
  w.bytes = w.enc + w.z + w.lse + w.part;
  return w;
}

template <int D, int MP, int NS>
cudaError_t launch_comm_tc_t(const CUtensorMap& tk, const CUtensorMap& tq, const CommArgs& a, int BH,
                             cudaStream_t st) {
  using C = CommCfg<D, MP, NS>;
  auto kern = comm_tc_kernel<D, MP, NS>;
  static cudaError_t attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (attr != cudaSuccess) return attr;
  kern<<<dim3(a.splits, C::kHalves, BH), C::kThreads, C::kSmemBytes, st>>>(tk, tq, a);
  return cudaGetLastError();
}

template <int MP>
cudaError_t launch_comm_tc_m(int D, const CUtensorMap& tk, const CUtensorMap& tq, const CommArgs& a, int BH,
                             cudaStream_t st) {
  switch (D) {
    case 16: return launch_comm_tc_t<16, MP, 4>(tk, tq, a, BH, st);
    case 32: return launch_comm_tc_t<32, MP, 4>(tk, tq, a, BH, st);
    default: return launch_comm_tc_t<64, MP, 3>(tk, tq, a, BH, st);
  }
}

int run_comm_tc(const void* Q, int q_batched, const void* K, void* C, int B, int H, int64_t N, int M, int D,
                bool f32_out, char* ws, cudaStream_t st, int* launches) {
  const int BH = B * H;
  const CommTcWs w = comm_tc_ws_layout(B, H, N, M, D);
  float* Ztmp = reinterpret_cast<float*>(ws + w.enc);
  float* lse2 = reinterpret_cast<float*>(ws + w.enc + w.z);
  float* part = reinterpret_cast<float*>(ws + w.enc + w.z + w.lse);
  int rc = run_encode(Q, q_batched, K, K, Ztmp, B, H, N, M, D, FLARE_BF16, ws, st, launches, false, lse2, true);
  if (rc) return rc;
  int* status = status_ptr();
  if (!status) return FLARE_ERR_CUDA;
  CUtensorMap tk, tq;
  if (!make_map(&tk, K, D, N, BH, kTileN) || !make_map(&tq, Q, D, M, q_batched ? BH : H, kLatRows))
    return FLARE_ERR_CUDA;
  CommArgs a;
  a.N = static_cast<int>(N);
  a.M = M;
  a.H = H;
  a.q_batched = q_batched;
  a.splits = w.splits;
  a.tiles = static_cast<int>(ceil_div(N, kTileN));
  a.lse2 = lse2;
  a.C_part = part;
  a.status = status;
  a.wait_ns = static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull;
  cudaError_t e;
  {
    ProfScope prof(FLARE_KERNEL_COMM_TC, st);
    e = M > kLatRows ? launch_comm_tc_m<256>(D, tk, tq, a, BH, st) : launch_comm_tc_m<128>(D, tk, tq, a, BH, st);
  }
  if (e != cudaSuccess) return FLARE_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>(ceil_div(int64_t(M) * M, 256)), BH);
  {
    ProfScope prof(FLARE_KERNEL_COMM_REDUCE, st);
    if (f32_out)
      comm_reduce_kernel<float><<<grid, 256, 0, st>>>(part, static_cast<float*>(C), M, w.splits);
    else
      comm_reduce_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(part, static_cast<__nv_bfloat16*>(C), M, w.splits);
  }
  if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_CUDA;
  *launches += 2;
  return FLARE_OK;
}

// The one-pass tensor-core form covers bf16 inputs with M % 16 == 0 and D <= 64.
bool comm_on_tensor_cores(int M, int D, int dtype) {
  return (dtype == FLARE_BF16 || dtype == FLARE_BF16_F32OUT) && M % 16 == 0 && D <= 64;
}

// ------------------------------------------------------------------ host-resident inputs
// flarepp_mix_host streams (b, h) chunks through the GPU: the copy of chunk
// c + 1 in, the mix of chunk c and the copy of chunk c - 1 out run at once on
// two copy streams and the caller's stream, with two device slots per chunk
// buffer.  One stream pair and one set of events per device, created once;
// calls are serialised by a mutex while they enqueue.
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t ev_in[2], ev_comp[2], ev_out[2], ev_seeds;
};

std::mutex g_pipe_mu;

HostPipe* host_pipe() {
  static HostPipe pipes[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  HostPipe& p = pipes[dev];
  if (!p.ready) {
    if (cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    for (int i = 0; i < 2; ++i)
      if (cudaEventCreateWithFlags(&p.ev_in[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.ev_comp[i], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.ev_out[i], cudaEventDisableTiming) != cudaSuccess)
        return nullptr;
    if (cudaEventCreateWithFlags(&p.ev_seeds, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    p.ready = true;
  }
  return &p;
}

struct HostWs {
  size_t seeds, chunk_in, chunk_out, mix, bytes;
};

HostWs host_ws_layout(int H, int64_t N, int M, int D, int dtype) {
  const size_t in_es = dtype == FLARE_F32 ? 4 : 2;
  const size_t out_es = dtype == FLARE_BF16 ? 2 : 4;
  HostWs w;
  w.seeds = align256(static_cast<size_t>(H) * M * D * in_es);
  w.chunk_in = align256(static_cast<size_t>(N) * D * in_es);
  w.chunk_out = align256(static_cast<size_t>(N) * D * out_es);
  w.mix = mix_ws_bytes(1, 1, N, M, D, dtype);
  w.bytes = w.seeds + 2 * (2 * w.chunk_in + w.chunk_out) + w.mix;
  return w;
}

bool host_ptr(const void* p) {
  if (!p) return false;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return true;  // not known to CUDA: pageable host memory
  }
  return attr.type == cudaMemoryTypeHost || attr.type == cudaMemoryTypeUnregistered;
}

// ------------------------------------------------------------------ backward
// Workspace of flarepp_mix_backward, in order: the encode's own workspace,
// Q_dyn and Z (dtype), lse1, lse2, c1, c2 ([BH][M] fp32), dZ, dQ_dyn
// ([BH][M][D] fp32), lse3, delta ([BH][N] fp32), two partial blocks
// [BH][S][M][D] fp32.
struct BackwardWs {
  char* enc;
  void* Qd;
  void* Z;
  float *lse1, *lse2, *c1, *c2, *dZ, *dQd, *lse3, *delta, *part;
  __nv_bfloat16 *dZ16, *dQd16;
  long long part_stride;
  int S;
  size_t bytes;
};

int backward_splits(int BH, int64_t N, int M) {
  const int64_t tiles = ceil_div(N, kBwdChunk);
  const int64_t chunks = ceil_div(M, kBwdChunk);
  const int64_t want = ceil_div(int64_t(2) * sm_count(), int64_t(BH) * chunks);
  return static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(want, tiles)));
}

// The backward's tensor-core kernels: bf16, D <= 64.
bool backward_tc(int D, int dtype) { return dtype == FLARE_BF16 && D <= 64; }

// Token splits of the latent-side kernels (the partial blocks' S).
int backward_latent_splits(int BH, int64_t N, int M, int D, int dtype) {
  // two CTAs per SM (256 TMEM columns each)
  if (backward_tc(D, dtype)) return choose_splits(BH * static_cast<int>(ceil_div(M, 128)), N, kBltcTok, 2);
  return backward_splits(BH, N, M);
}

BackwardWs backward_ws_layout(char* base, int BH, int64_t N, int M, int D, int dtype) {
  BackwardWs w;
  const size_t esz = dtype == FLARE_BF16 ? 2 : 4;
  const size_t lat = static_cast<size_t>(BH) * M;
  w.S = backward_latent_splits(BH, N, M, D, dtype);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  w.enc = take(encode_ws_layout(nullptr, BH, N, M, D, dtype).bytes);
  w.Qd = take(lat * D * esz);
  w.Z = take(lat * D * esz);
  w.lse1 = reinterpret_cast<float*>(take(lat * 4));
  w.lse2 = reinterpret_cast<float*>(take(lat * 4));
  w.c1 = reinterpret_cast<float*>(take(lat * 4));
  w.c2 = reinterpret_cast<float*>(take(lat * 4));
  w.dZ = reinterpret_cast<float*>(take(lat * D * 4));
  w.dQd = reinterpret_cast<float*>(take(lat * D * 4));
  w.dZ16 = reinterpret_cast<__nv_bfloat16*>(take(lat * D * 2));
  w.dQd16 = reinterpret_cast<__nv_bfloat16*>(take(lat * D * 2));
  w.lse3 = reinterpret_cast<float*>(take(static_cast<size_t>(BH) * N * 4));
  w.delta = reinterpret_cast<float*>(take(static_cast<size_t>(BH) * N * 4));
  w.part_stride = static_cast<long long>(BH) * w.S * M * D;
  w.part = reinterpret_cast<float*>(take(2 * static_cast<size_t>(w.part_stride) * 4));
  w.bytes = off;
  return w;
}

template <typename K>
cudaError_t launch_dyn(K kernel, dim3 grid, int smem, cudaStream_t st, const BwdArgs& a) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kBwdThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D, int MODE>
cudaError_t launch_latent_grad_tc(const BwdArgs& a, const BackwardWs& w, int BH, cudaStream_t st) {
  constexpr int kMode = MODE == kBwdDec ? 0 : 1;
  using C = BltcCfg<D, kMode>;
  CUtensorMap mA, mB, mK, mX;
  const int64_t N = a.N;
  const void* A = MODE == kBwdEncSeed ? a.seeds : w.Qd;
  const void* Bm = MODE == kBwdDec ? w.Z : (MODE == kBwdEncRouting ? static_cast<const void*>(w.dZ16) : w.dQd16);
  const void* X = MODE == kBwdDec ? a.dY : a.V;
  if (!make_map(&mA, A, D, a.M, MODE == kBwdEncSeed ? a.H : BH, 128) || !make_map(&mB, Bm, D, a.M, BH, 128) ||
      !make_map(&mK, a.K, D, N, BH, kBltcTok) || !make_map(&mX, X, D, N, BH, kBltcTok))
    return cudaErrorInvalidValue;
  BltcArgs t;
  t.N = a.N;
  t.M = a.M;
  t.S = a.S;
  t.tiles = static_cast<int>(ceil_div(N, kBltcTok));
  t.lse_row = MODE == kBwdEncSeed ? a.lse1 : a.lse2;
  t.c_row = MODE == kBwdEncSeed ? a.c1 : a.c2;
  t.lse3 = a.lse3;
  t.delta = a.delta;
  t.part = a.part;
  t.part_stride = a.part_stride;
  t.status = status_ptr();
  t.wait_ns = static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull;
  // at least 80 KB of shared memory: at most two CTAs per SM, each with 256 TMEM columns
  const int smem = C::kSmemBytes > 80 * 1024 ? C::kSmemBytes : 80 * 1024;
  auto kern = latent_grad_tc_kernel<D, kMode>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(a.S, BH, static_cast<unsigned>(ceil_div(a.M, 128))), C::kThreads, smem, st>>>(
      mA, mB, mK, mX, t, MODE == kBwdEncSeed ? 0 : 1, a.H);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_token_stats_tc(const BwdArgs& a, const BackwardWs& w, int BH, cudaStream_t st) {
  using C = BstCfg<D>;
  CUtensorMap mQd, mZ, mK, mdY;
  const int64_t N = a.N;
  if (!make_map(&mQd, w.Qd, D, a.M, BH, 64) || !make_map(&mZ, w.Z, D, a.M, BH, 64) ||
      !make_map(&mK, a.K, D, N, BH, 128) || !make_map(&mdY, a.dY, D, N, BH, 128))
    return cudaErrorInvalidValue;
  BstArgs t;
  t.N = a.N;
  t.M = a.M;
  t.tiles = static_cast<int>(ceil_div(N, 128));
  t.splits = choose_splits(BH, N, 128, 2);  // two CTAs per SM
  t.lse3 = a.lse3;
  t.delta = a.delta;
  t.status = status_ptr();
  t.wait_ns = static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull;
  // at least 80 KB of shared memory: at most two CTAs per SM, each with 256 TMEM columns
  const int smem = C::kSmemBytes > 80 * 1024 ? C::kSmemBytes : 80 * 1024;
  auto kern = token_stats_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(t.splits, BH), C::kThreads, smem, st>>>(mQd, mZ, mK, mdY, t);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_token_grad_tc(const BwdArgs& a, const BackwardWs& w, int BH, cudaStream_t st) {
  using C = BtcCfg<D>;
  CUtensorMap mQd, mZ, mdZ, mS, mdQ, mK, mdY, mV;
  const int64_t N = a.N;
  if (!make_map(&mQd, w.Qd, D, a.M, BH, kBtcChunk) || !make_map(&mZ, w.Z, D, a.M, BH, kBtcChunk) ||
      !make_map(&mdZ, w.dZ16, D, a.M, BH, kBtcChunk) || !make_map(&mS, a.seeds, D, a.M, a.H, kBtcChunk) ||
      !make_map(&mdQ, w.dQd16, D, a.M, BH, kBtcChunk) || !make_map(&mK, a.K, D, N, BH, kBtcTile) ||
      !make_map(&mdY, a.dY, D, N, BH, kBtcTile) || !make_map(&mV, a.V, D, N, BH, kBtcTile))
    return cudaErrorInvalidValue;
  BwdTcArgs t;
  t.N = a.N;
  t.M = a.M;
  t.H = a.H;
  t.tiles = static_cast<int>(ceil_div(N, kBtcTile));
  t.splits = choose_splits(BH, N, kBtcTile);
  t.lse1 = a.lse1;
  t.lse2 = a.lse2;
  t.c1 = a.c1;
  t.c2 = a.c2;
  t.lse3 = a.lse3;
  t.delta = a.delta;
  t.dK = static_cast<__nv_bfloat16*>(a.dK);
  t.dV = static_cast<__nv_bfloat16*>(a.dV);
  t.status = status_ptr();
  t.wait_ns = static_cast<unsigned long long>(g_wait_ms.load()) * 1000000ull;
  // at least 120 KB of shared memory: one CTA per SM, so two CTAs never
  // contend for the 512 TMEM columns each allocates
  const int smem = C::kSmemBytes > 120 * 1024 ? C::kSmemBytes : 120 * 1024;
  auto kern = token_grad_tc_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(t.splits, BH), C::kThreads, smem, st>>>(mQd, mZ, mdZ, mS, mdQ, mK, mdY, mV, t);
  return cudaGetLastError();
}

// phase < 0: the whole backward, each reduction in one kernel.  phase 0..3:
// one phase of a token-sharded backward; between phases the caller sums
// a.exch over the ranks (phase 0 leaves dZ and the decode part of dQ_dyn
// there, phase 1 the routing part of dQ_dyn, phase 2 d_seeds in fp32).  A
// shard without tokens (a.N == 0) contributes zeros.
template <int D, typename T>
cudaError_t launch_backward_d(const BwdArgs& a, const BackwardWs& w, int B, int BH, int dtype, cudaStream_t st,
                              int phase = -1) {
  const unsigned tok_tiles = static_cast<unsigned>(ceil_div(static_cast<int64_t>(a.N), kBwdChunk));
  const unsigned lat_chunks = static_cast<unsigned>(ceil_div(a.M, kBwdChunk));
  const dim3 red(static_cast<unsigned>(ceil_div(a.M, 8)), BH);
  const bool all = phase < 0;
  const bool tokens = a.N > 0;
  cudaError_t e = cudaSuccess;
  const bool tc = D <= 64 && backward_tc(D, dtype);
  // one latent-side pass: the tensor-core kernel or the CUDA-core one
  auto latent = [&](auto mode) -> cudaError_t {
    constexpr int kMode = decltype(mode)::value;
    ProfScope prof(FLARE_KERNEL_BWD_LATENT, st);
    if constexpr (D <= 64) {
      if (tc) return launch_latent_grad_tc<D, kMode>(a, w, BH, st);
    }
    return launch_dyn(latent_grad_kernel<D, T, kMode>, dim3(a.S, BH, lat_chunks), bwd_smem_latent<D>(), st, a);
  };
  auto reduce = [&](auto mode, auto stage, dim3 grid) -> cudaError_t {
    ProfScope prof(FLARE_KERNEL_BWD_REDUCE, st);
    grad_reduce_kernel<D, T, decltype(mode)::value, decltype(stage)::value><<<grid, kBwdThreads, 0, st>>>(a, B);
    return cudaGetLastError();
  };
  // this rank's sums: the reduction of its partials, or zeros without tokens
  auto local = [&](auto mode, dim3 grid, size_t floats) -> cudaError_t {
    if (!tokens) return cudaMemsetAsync(a.exch, 0, floats * sizeof(float), st);
    return reduce(mode, std::integral_constant<int, kStageLocal>{}, grid);
  };
  using Dec = std::integral_constant<int, kBwdDec>;
  using Rout = std::integral_constant<int, kBwdEncRouting>;
  using Seed = std::integral_constant<int, kBwdEncSeed>;
  using Fused = std::integral_constant<int, kStageFused>;
  using Finish = std::integral_constant<int, kStageFinish>;
  const size_t L = static_cast<size_t>(BH) * a.M * D;
  if (all || phase == 0) {
    if (tokens) {
      ProfScope prof(FLARE_KERNEL_BWD_TOKEN_STATS, st);
      if constexpr (D <= 64) {
        if (tc) e = launch_token_stats_tc<D>(a, w, BH, st);
      }
      if (!tc) e = launch_dyn(token_stats_kernel<D, T>, dim3(tok_tiles, BH), bwd_smem_token_stats<D>(), st, a);
    }
    if (e) return e;
    if (tokens && (e = latent(Dec{}))) return e;
    if ((e = all ? reduce(Dec{}, Fused{}, red) : local(Dec{}, red, 2 * L))) return e;
  }
  if (all || phase == 1) {
    if (!all && (e = reduce(Dec{}, Finish{}, red))) return e;
    if (tokens && (e = latent(Rout{}))) return e;
    if ((e = all ? reduce(Rout{}, Fused{}, red) : local(Rout{}, red, L))) return e;
  }
  if (all || phase == 2) {
    if (!all && (e = reduce(Rout{}, Finish{}, red))) return e;
    if (tokens && (e = latent(Seed{}))) return e;
    const dim3 sred(red.x, a.H);
    if ((e = all ? reduce(Seed{}, Fused{}, sred) : local(Seed{}, sred, static_cast<size_t>(a.H) * a.M * D))) return e;
  }
  if (all || phase == 3) {
    if (!all && (e = reduce(Seed{}, Finish{}, dim3(red.x, a.H)))) return e;
    if (!tokens) return cudaSuccess;
    ProfScope prof(FLARE_KERNEL_BWD_TOKEN_GRAD, st);
    if constexpr (D <= 64) {
      if (tc) return launch_token_grad_tc<D>(a, w, BH, st);
    }
    return launch_dyn(token_grad_kernel<D, T>, dim3(tok_tiles, BH), bwd_smem_token_grad<D>(), st, a);
  }
  return cudaSuccess;
}

template <typename T>
cudaError_t launch_backward_t(int D, const BwdArgs& a, const BackwardWs& w, int B, int BH, int dtype,
                              cudaStream_t st, int phase) {
  switch (D) {
    case 16: return launch_backward_d<16, T>(a, w, B, BH, dtype, st, phase);
    case 32: return launch_backward_d<32, T>(a, w, B, BH, dtype, st, phase);
    case 64: return launch_backward_d<64, T>(a, w, B, BH, dtype, st, phase);
    default: return launch_backward_d<128, T>(a, w, B, BH, dtype, st, phase);
  }
}

// What flarepp_mix_save keeps for the backward, in order, each region
// 256-byte aligned: Q_dyn [B][H][M][D] and Z (dtype), lse1 and lse2
// [B][H][M] fp32 (the two encodes' log-sum-exps, natural log).
struct SavedLayout {
  void* Qd;
  void* Z;
  float* lse1;
  float* lse2;
  size_t bytes;
};

SavedLayout saved_layout(void* base, int BH, int M, int D, int dtype) {
  SavedLayout l;
  const size_t lat = static_cast<size_t>(BH) * M;
  const size_t esz = dtype == FLARE_BF16 ? 2 : 4;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* q = p ? p + off : nullptr;
    off += align256(bytes);
    return q;
  };
  l.Qd = take(lat * D * esz);
  l.Z = take(lat * D * esz);
  l.lse1 = reinterpret_cast<float*>(take(lat * 4));
  l.lse2 = reinterpret_cast<float*>(take(lat * 4));
  l.bytes = off;
  return l;
}

int run_backward(const void* seeds, const void* K, const void* V, const void* dY, void* d_seeds, void* dK, void* dV,
                 int B, int H, int64_t N, int M, int D, int dtype, char* ws, cudaStream_t st, int* launches,
                 void* saved = nullptr, int phase = -1, float* exch = nullptr) {
  const int BH = B * H;
  BackwardWs w = backward_ws_layout(ws, BH, N, M, D, dtype);
  if (saved) {
    // Q_dyn, Z and the encodes' log-sum-exps as flarepp_mix_save kept them
    const SavedLayout l = saved_layout(saved, BH, M, D, dtype);
    w.Qd = l.Qd;
    w.Z = l.Z;
    w.lse1 = l.lse1;
    w.lse2 = l.lse2;
  } else {
    // the forward's encodes again, for Q_dyn and Z as it stored them and
    // their per-latent log-sum-exps
    int rc = run_encode(seeds, 0, K, V, w.Qd, B, H, N, M, D, dtype, w.enc, st, launches, false, w.lse1);
    if (rc) return rc;
    rc = run_encode(w.Qd, 1, K, V, w.Z, B, H, N, M, D, dtype, w.enc, st, launches, false, w.lse2);
    if (rc) return rc;
  }
  BwdArgs a;
  a.N = static_cast<int>(N);
  a.M = M;
  a.H = H;
  a.seeds = seeds;
  a.K = K;
  a.V = V;
  a.dY = dY;
  a.Qd = w.Qd;
  a.Z = w.Z;
  a.lse1 = w.lse1;
  a.lse2 = w.lse2;
  a.lse3 = w.lse3;
  a.delta = w.delta;
  a.dZ = w.dZ;
  a.dQd = w.dQd;
  a.c1 = w.c1;
  a.c2 = w.c2;
  const bool tc = backward_tc(D, dtype);
  a.dZ16 = tc ? w.dZ16 : nullptr;
  a.dQd16 = tc ? w.dQd16 : nullptr;
  a.part = w.part;
  a.part_stride = w.part_stride;
  a.S = w.S;
  a.d_seeds = d_seeds;
  a.dK = dK;
  a.dV = dV;
  a.exch = exch;
  const cudaError_t e = dtype == FLARE_BF16 ? launch_backward_t<__nv_bfloat16>(D, a, w, B, BH, dtype, st, phase)
                                            : launch_backward_t<float>(D, a, w, B, BH, dtype, st, phase);
  *launches += phase < 0 ? 8 : 3;
  return e == cudaSuccess ? FLARE_OK : FLARE_ERR_CUDA;
}

// Self-test of the bounded wait every kernel uses: one warp waits on an
// mbarrier that nothing arrives at.  ptx::mbar_wait gives up after limit_ns
// (%globaltimer), and the kernel records FLARE_ERR_TIMEOUT with its site in
// the device status word and returns, as the real kernels do on a timeout.
// No TMA copy, MMA or TMEM is involved, so nothing else has to drain.
constexpr int kSiteWaitProbe = 13;

__global__ void __launch_bounds__(32) wait_probe_kernel(int* status, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
  }
  __syncwarp();
  const bool ok = ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns);  // phase 0 never completes
  if (!ok && threadIdx.x == 0) record_error(status, kErrTimeout, kSiteWaitProbe);
}

// fp32 tensor in device memory with 4-byte alignment (the per-latent
// statistics of a slice of a gathered [R][B][H][M] array need no more).
bool device_ptr_f32(const void* p) {
  if (!p || (reinterpret_cast<uintptr_t>(p) & 3u)) return false;
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return attr.type == cudaMemoryTypeDevice || attr.type == cudaMemoryTypeManaged;
}

// A token shard with no tokens: O = 0, lse = -inf (it then carries no weight).
__global__ void empty_shard_kernel(float* O, float* lse, size_t rows, int D) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < rows * D) O[i] = 0.f;
  if (i < rows) lse[i] = -INFINITY;
}

extern "C" {

size_t flare_encode_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (check_sizes(B, H, N, M, D, dtype)) return 0;
  return encode_ws_layout(nullptr, B * H, N, M, D, dtype).bytes;
}

size_t flarepp_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (check_sizes(B, H, N, M, D, dtype)) return 0;
  return mix_ws_bytes(B, H, N, M, D, dtype);
}

int flare_encode(const void* Q, int q_batched, const void* K, const void* V, void* Z, int B, int H, int64_t N,
                 int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (q_batched != 0 && q_batched != 1) return FLARE_ERR_INVALID_ARG;
  if (!device_ptr(Q) || !device_ptr(K) || !device_ptr(V) || !device_ptr(Z)) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes, encode_ws_layout(nullptr, B * H, N, M, D, dtype).bytes, st, &s);
  if (rc) return rc;
  int launches = 0;
  rc = run_encode(Q, q_batched, K, V, Z, B, H, N, M, D, dtype, s.ptr, st, &launches);
  const int rc2 = release_scratch(s, st);
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

size_t flare_encode_lse_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (N <= 0) return 0;  // an empty shard needs none
  if (check_sizes(B, H, N, M, D, dtype)) return 0;
  return encode_ws_layout(nullptr, B * H, N, M, D, dtype).bytes;
}

int flare_encode_lse(const void* Q, int q_batched, const void* K, const void* V, float* O, float* lse, int B,
                     int H, int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes,
                     void* stream) {
  SplitPin pin;
  if (N < 0) return FLARE_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, N == 0 ? 1 : N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (q_batched != 0 && q_batched != 1) return FLARE_ERR_INVALID_ARG;
  if (!device_ptr(Q) || !device_ptr(O) || !device_ptr_f32(lse)) return FLARE_ERR_INVALID_ARG;
  if (N > 0 && (!device_ptr(K) || !device_ptr(V))) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (N == 0) {
    const size_t rows = static_cast<size_t>(B) * H * M;
    empty_shard_kernel<<<static_cast<unsigned>(ceil_div(static_cast<int64_t>(rows * D), 256)), 256, 0, st>>>(
        O, lse, rows, D);
    if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_CUDA;
    t_last_launches = 1;
    return FLARE_OK;
  }
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes, encode_ws_layout(nullptr, B * H, N, M, D, dtype).bytes, st, &s);
  if (rc) return rc;
  int launches = 0;
  rc = run_encode(Q, q_batched, K, V, O, B, H, N, M, D, dtype, s.ptr, st, &launches, false, lse, true);
  const int rc2 = release_scratch(s, st);
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

int flare_lse_combine(const float* O_parts, const float* lse_parts, int R, int64_t part_stride, void* out,
                      float* lse_out, int B, int H, int M, int D, int dtype, void* stream) {
  int rc = check_sizes(B, H, 1, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (R < 1 || part_stride < 0) return FLARE_ERR_INVALID_ARG;
  if (!device_ptr(O_parts) || !device_ptr_f32(lse_parts) || !device_ptr(out)) return FLARE_ERR_INVALID_ARG;
  if (lse_out && !device_ptr_f32(lse_out)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int BH = B * H;
  const long long rows = static_cast<long long>(BH) * M;
  const MergeGeom g{R, M, D, static_cast<long long>(M) * D, part_stride ? part_stride : rows * D, M,
                    part_stride ? part_stride : rows};
  const dim3 grid(static_cast<unsigned>(ceil_div(int64_t(M) * D, 256)), BH);
  ProfScope prof(FLARE_KERNEL_MERGE, st);
  if (dtype == FLARE_BF16)
    lse_merge_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(O_parts, lse_parts, nullptr,
                                                               static_cast<__nv_bfloat16*>(out), lse_out, g);
  else
    lse_merge_kernel<float, true><<<grid, 256, 0, st>>>(O_parts, lse_parts, nullptr, static_cast<float*>(out),
                                                       lse_out, g);
  if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_CUDA;
  t_last_launches = 1;
  return FLARE_OK;
}

size_t flarepp_mix_backward_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (check_sizes(B, H, N, M, D, dtype) || dtype == FLARE_BF16_F32OUT) return 0;
  return backward_ws_layout(nullptr, B * H, N, M, D, dtype).bytes;
}

int flarepp_mix_backward(const void* seeds, const void* K, const void* V, const void* dY, void* d_seeds, void* dK,
                         void* dV, int B, int H, int64_t N, int M, int D, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  for (const void* p : {seeds, K, V, dY, static_cast<const void*>(d_seeds), static_cast<const void*>(dK),
                        static_cast<const void*>(dV)})
    if (!device_ptr(p)) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes, backward_ws_layout(nullptr, B * H, N, M, D, dtype).bytes, st, &s);
  if (rc) return rc;
  int launches = 0;
  rc = run_backward(seeds, K, V, dY, d_seeds, dK, dV, B, H, N, M, D, dtype, s.ptr, st, &launches);
  const int rc2 = release_scratch(s, st);
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

size_t flarepp_saved_bytes(int B, int H, int M, int D, int dtype) {
  if (check_sizes(B, H, 1, M, D, dtype) || dtype == FLARE_BF16_F32OUT) return 0;
  return saved_layout(nullptr, B * H, M, D, dtype).bytes;
}

int flarepp_mix_save(const void* seeds, const void* K, const void* V, void* Y, void* saved, int B, int H, int64_t N,
                     int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (!device_ptr(saved)) return FLARE_ERR_INVALID_ARG;
  const SavedLayout l = saved_layout(saved, B * H, M, D, dtype);
  return mix_impl(seeds, K, V, Y, l.Qd, l.Z, B, H, N, M, D, dtype, workspace, workspace_bytes, stream, l.lse1, l.lse2);
}

int flarepp_mix_backward_saved(const void* seeds, const void* K, const void* V, const void* dY, const void* saved,
                               void* d_seeds, void* dK, void* dV, int B, int H, int64_t N, int M, int D, int dtype,
                               void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  for (const void* p : {seeds, K, V, dY, saved, static_cast<const void*>(d_seeds), static_cast<const void*>(dK),
                        static_cast<const void*>(dV)})
    if (!device_ptr(p)) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes, backward_ws_layout(nullptr, B * H, N, M, D, dtype).bytes, st, &s);
  if (rc) return rc;
  int launches = 0;
  rc = run_backward(seeds, K, V, dY, d_seeds, dK, dV, B, H, N, M, D, dtype, s.ptr, st, &launches,
                    const_cast<void*>(saved));
  const int rc2 = release_scratch(s, st);
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

size_t flarepp_backward_shard_exchange_floats(int B, int H, int M, int D) {
  if (B < 1 || H < 1 || M < 1 || D < 1) return 0;
  return 2 * static_cast<size_t>(B) * H * M * D;
}

size_t flarepp_backward_shard_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (N < 0 || check_sizes(B, H, N == 0 ? 1 : N, M, D, dtype) || dtype == FLARE_BF16_F32OUT) return 0;
  return backward_ws_layout(nullptr, B * H, N, M, D, dtype).bytes;
}

int flarepp_mix_backward_shard(int phase, const void* seeds, const void* K, const void* V, const void* dY,
                               const void* saved, float* exchange, void* d_seeds, void* dK, void* dV, int B, int H,
                               int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes,
                               void* stream) {
  SplitPin pin;
  if (phase < 0 || phase > 3 || N < 0) return FLARE_ERR_INVALID_ARG;
  int rc = check_sizes(B, H, N == 0 ? 1 : N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (!device_ptr(seeds) || !device_ptr(saved) || !device_ptr(exchange) || !device_ptr(d_seeds))
    return FLARE_ERR_INVALID_ARG;
  if (N > 0 && (!device_ptr(K) || !device_ptr(V) || !device_ptr(dY) || !device_ptr(dK) || !device_ptr(dV)))
    return FLARE_ERR_INVALID_ARG;
  // the workspace carries the state between the four phases: it is the caller's
  if (!device_ptr(workspace) ||
      workspace_bytes < backward_ws_layout(nullptr, B * H, N, M, D, dtype).bytes)
    return FLARE_ERR_INVALID_ARG;
  int launches = 0;
  rc = run_backward(seeds, K, V, dY, d_seeds, dK, dV, B, H, N, M, D, dtype, static_cast<char*>(workspace),
                    static_cast<cudaStream_t>(stream), &launches, const_cast<void*>(saved), phase, exchange);
  if (!rc) t_last_launches = launches;
  return rc;
}

int flare_decode(const void* K, const void* Q, int q_batched, const void* Z, void* Y, int B, int H, int64_t N,
                 int M, int D, int dtype, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (q_batched != 0 && q_batched != 1) return FLARE_ERR_INVALID_ARG;
  if (!device_ptr(K) || !device_ptr(Q) || !device_ptr(Z) || !device_ptr(Y)) return FLARE_ERR_INVALID_ARG;
  int launches = 0;
  rc = run_decode(K, Q, q_batched, Z, Y, B, H, N, M, D, dtype, static_cast<cudaStream_t>(stream), &launches);
  if (!rc) t_last_launches = launches;
  return rc;
}

int flarepp_mix(const void* seeds, const void* K, const void* V, void* Y, int B, int H, int64_t N, int M, int D,
                int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  return mix_impl(seeds, K, V, Y, nullptr, nullptr, B, H, N, M, D, dtype, workspace, workspace_bytes, stream);
}

int flarepp_mix_debug(const void* seeds, const void* K, const void* V, void* Y, void* Q_dyn, void* Z, int B, int H,
                      int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  if (!Q_dyn || !Z) return FLARE_ERR_INVALID_ARG;
  return mix_impl(seeds, K, V, Y, Q_dyn, Z, B, H, N, M, D, dtype, workspace, workspace_bytes, stream);
}

size_t flare_communication_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (check_sizes(B, H, N, M, D, dtype)) return 0;
  if (comm_on_tensor_cores(M, D, dtype)) return comm_tc_ws_layout(B, H, N, M, D).bytes;
  if (dtype == FLARE_BF16_F32OUT) return 0;
  return comm_ws_layout(B, H, N, M, D, dtype).bytes;
}

int flare_communication_matrix(const void* Q, int q_batched, const void* K, void* C, int B, int H, int64_t N, int M,
                               int D, int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  const bool tc = comm_on_tensor_cores(M, D, dtype);
  if (dtype == FLARE_BF16_F32OUT && !tc) return FLARE_ERR_UNSUPPORTED;
  if (q_batched != 0 && q_batched != 1) return FLARE_ERR_INVALID_ARG;
  if (!device_ptr(Q) || !device_ptr(K) || !device_ptr(C)) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes,
                   tc ? comm_tc_ws_layout(B, H, N, M, D).bytes : comm_ws_layout(B, H, N, M, D, dtype).bytes, st, &s);
  if (rc) return rc;
  int launches = 0;
  if (tc)
    rc = run_comm_tc(Q, q_batched, K, C, B, H, N, M, D, dtype == FLARE_BF16_F32OUT, s.ptr, st, &launches);
  else
    rc = dtype == FLARE_BF16 ? run_comm<__nv_bfloat16>(Q, q_batched, K, C, B, H, N, M, D, dtype, s.ptr, st, &launches)
                             : run_comm<float>(Q, q_batched, K, C, B, H, N, M, D, dtype, s.ptr, st, &launches);
  const int rc2 = release_scratch(s, st);
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

size_t flarepp_mix_host_workspace_size(int B, int H, int64_t N, int M, int D, int dtype) {
  SplitPin pin;
  if (check_sizes(B, H, N, M, D, dtype)) return 0;
  return host_ws_layout(H, N, M, D, dtype).bytes;
}

int flarepp_mix_host(const void* seeds, const void* K, const void* V, void* Y, int B, int H, int64_t N, int M, int D,
                     int dtype, void* workspace, size_t workspace_bytes, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (!host_ptr(seeds) || !host_ptr(K) || !host_ptr(V) || !host_ptr(Y)) return FLARE_ERR_INVALID_ARG;
  if (workspace && !device_ptr(workspace)) return FLARE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_pipe_mu);
  HostPipe* pipe = host_pipe();
  if (!pipe) return FLARE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const HostWs w = host_ws_layout(H, N, M, D, dtype);
  Scratch s;
  rc = get_scratch(workspace, workspace_bytes, w.bytes, st, &s);
  if (rc) return rc;
  // the copy streams start after the caller's earlier work (workspace reuse)
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  bool good = ok(cudaEventRecord(pipe->ev_seeds, st)) && ok(cudaStreamWaitEvent(pipe->in, pipe->ev_seeds, 0)) &&
              ok(cudaStreamWaitEvent(pipe->out, pipe->ev_seeds, 0));
  const size_t in_es = dtype == FLARE_F32 ? 4 : 2;
  const size_t out_es = dtype == FLARE_BF16 ? 2 : 4;
  const size_t in_bytes = static_cast<size_t>(N) * D * in_es, out_bytes = static_cast<size_t>(N) * D * out_es;
  char* seeds_d = s.ptr;
  char* slot_base[2] = {s.ptr + w.seeds, s.ptr + w.seeds + 2 * w.chunk_in + w.chunk_out};
  char* mix_ws = s.ptr + w.seeds + 2 * (2 * w.chunk_in + w.chunk_out);
  good = good && ok(cudaMemcpyAsync(seeds_d, seeds, static_cast<size_t>(H) * M * D * in_es, cudaMemcpyHostToDevice,
                                    pipe->in)) &&
         ok(cudaEventRecord(pipe->ev_seeds, pipe->in)) && ok(cudaStreamWaitEvent(st, pipe->ev_seeds, 0));
  int launches = 0;
  const int chunks = B * H;
  for (int c = 0; good && !rc && c < chunks; ++c) {
    const int sl = c & 1, h = c % H;
    char* Kd = slot_base[sl];
    char* Vd = Kd + w.chunk_in;
    char* Yd = Vd + w.chunk_in;
    const char* Kh = static_cast<const char*>(K) + static_cast<size_t>(c) * in_bytes;
    const char* Vh = static_cast<const char*>(V) + static_cast<size_t>(c) * in_bytes;
    char* Yh = static_cast<char*>(Y) + static_cast<size_t>(c) * out_bytes;
    // in: once the mix of chunk c - 2 has read this slot
    if (c >= 2) good = ok(cudaStreamWaitEvent(pipe->in, pipe->ev_comp[sl], 0));
    good = good && ok(cudaMemcpyAsync(Kd, Kh, in_bytes, cudaMemcpyHostToDevice, pipe->in)) &&
           ok(cudaMemcpyAsync(Vd, Vh, in_bytes, cudaMemcpyHostToDevice, pipe->in)) &&
           ok(cudaEventRecord(pipe->ev_in[sl], pipe->in));
    // mix: once the inputs are in and Y of chunk c - 2 has left this slot
    good = good && ok(cudaStreamWaitEvent(st, pipe->ev_in[sl], 0)) &&
           (c < 2 || ok(cudaStreamWaitEvent(st, pipe->ev_out[sl], 0)));
    if (!good) break;
    rc = mix_impl(seeds_d + static_cast<size_t>(h) * M * D * in_es, Kd, Vd, Yd, nullptr, nullptr, 1, 1, N, M, D,
                  dtype, mix_ws, w.mix, st);
    launches += t_last_launches;
    // out: once the mix is done
    good = good && !rc && ok(cudaEventRecord(pipe->ev_comp[sl], st)) &&
           ok(cudaStreamWaitEvent(pipe->out, pipe->ev_comp[sl], 0)) &&
           ok(cudaMemcpyAsync(Yh, Yd, out_bytes, cudaMemcpyDeviceToHost, pipe->out)) &&
           ok(cudaEventRecord(pipe->ev_out[sl], pipe->out));
  }
  // the caller's stream completes after every copy out
  for (int sl = 0; good && sl < 2 && sl < chunks; ++sl) good = ok(cudaStreamWaitEvent(st, pipe->ev_out[sl], 0));
  const int rc2 = release_scratch(s, st);
  if (!rc && !good) rc = FLARE_ERR_CUDA;
  if (!rc) {
    rc = rc2;
    t_last_launches = launches;
  }
  return rc;
}

int flare_selftest_wait_timeout(int limit_ms, void* stream) {
  if (limit_ms < 1 || limit_ms > 1000) return FLARE_ERR_INVALID_ARG;
  int* status = status_ptr();
  if (!status) return FLARE_ERR_CUDA;
  wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      status, static_cast<unsigned long long>(limit_ms) * 1000000ull);
  if (cudaGetLastError() != cudaSuccess) return FLARE_ERR_CUDA;
  t_last_launches = 1;
  return FLARE_OK;
}

int flare_check_status(void* stream, int* site) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FLARE_ERR_CUDA;
  int* p = status_ptr();
  if (!p) return FLARE_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpy(h, p, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return FLARE_ERR_CUDA;
  const int zero[2] = {0, 0};
  if (cudaMemcpy(p, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return FLARE_ERR_CUDA;
  if (site) *site = h[1];
  return h[0];
}

const char* flare_status_string(int status) {
  switch (status) {
    case FLARE_OK: return "ok";
    case FLARE_ERR_INVALID_ARG: return "invalid argument";
    case FLARE_ERR_UNSUPPORTED: return "unsupported sizes";
    case FLARE_ERR_CUDA: return "CUDA error";
    case FLARE_ERR_TIMEOUT: return "kernel wait timed out";
    default: return "unknown status";
  }
}

int flare_last_launch_count(void) { return t_last_launches; }

const char* flare_cuda_error_string(void) { return cudaGetErrorString(cudaPeekAtLastError()); }

int flare_set_split_override(int splits) { return g_split_override.exchange(splits < 0 ? 0 : splits); }

int flare_encode_splits(int B, int H, int64_t N) {
  if (B < 1 || H < 1 || N < 1) return 0;
  return choose_splits(B * H, N, kEncTile);
}

int flare_set_wait_limit_ms(int ms) { return g_wait_ms.exchange(ms < 1 ? 1 : ms); }

int flare_set_launch_overlap(int mode) { return g_launch_overlap.exchange(mode < -1 ? -1 : (mode > 1 ? 1 : mode)); }

int flare_profile_begin(int max_launches) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (g_prof.on || max_launches < 1) return FLARE_ERR_INVALID_ARG;
  g_prof.ev.assign(2 * static_cast<size_t>(max_launches), nullptr);
  for (auto& e : g_prof.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (auto& x : g_prof.ev)
        if (x) cudaEventDestroy(x);
      g_prof.ev.clear();
      return FLARE_ERR_CUDA;
    }
  g_prof.kind.assign(max_launches, 0);
  g_prof.cap = max_launches;
  g_prof.used = 0;
  g_prof.on = true;
  return FLARE_OK;
}

int flare_profile_end(float* ms, int* kinds, int max_records) {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (!g_prof.on) return -FLARE_ERR_INVALID_ARG;
  int n = std::min(g_prof.used, max_records);
  int rc = n;
  for (int i = 0; i < g_prof.used; ++i) {
    if (cudaEventSynchronize(g_prof.ev[2 * i + 1]) != cudaSuccess) rc = -FLARE_ERR_CUDA;
    if (i < n && rc >= 0) {
      if (cudaEventElapsedTime(&ms[i], g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) != cudaSuccess) rc = -FLARE_ERR_CUDA;
      kinds[i] = g_prof.kind[i];
    }
  }
  for (auto& e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.on = false;
  g_prof.used = g_prof.cap = 0;
  return rc;
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation encode
// Scratch for flare_encode_noalloc: a fixed array in the library's own device
// image, so the entry point never allocates.  Host code must not use the
// symbol itself as a pointer (it is a host-side stand-in); the device address
// is looked up once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FLARE_NOALLOC_SCRATCH_BYTES];

namespace flare {
namespace {

char* noalloc_scratch() {
  static char* ptrs[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    ptrs[dev] = static_cast<char*>(p);
  }
  return ptrs[dev];
}

}  // namespace
}  // namespace flare

extern "C" int flare_encode_noalloc(const void* Q, int q_batched, const void* K, const void* V, void* Z, int B,
                                    int H, int64_t N, int M, int D, int dtype, void* stream) {
  SplitPin pin;
  int rc = check_sizes(B, H, N, M, D, dtype);
  if (rc) return rc;
  if (dtype == FLARE_BF16_F32OUT) return FLARE_ERR_UNSUPPORTED;
  if (q_batched != 0 && q_batched != 1) return FLARE_ERR_INVALID_ARG;
  if (!device_ptr(Q) || !device_ptr(K) || !device_ptr(V) || !device_ptr(Z)) return FLARE_ERR_INVALID_ARG;
  if (encode_ws_layout(nullptr, B * H, N, M, D, dtype).bytes > FLARE_NOALLOC_SCRATCH_BYTES)
    return FLARE_ERR_UNSUPPORTED;
  char* ws = noalloc_scratch();
  if (!ws) return FLARE_ERR_CUDA;
  int launches = 0;
  rc = run_encode(Q, q_batched, K, V, Z, B, H, N, M, D, dtype, ws, static_cast<cudaStream_t>(stream), &launches);
  if (!rc) t_last_launches = launches;
  return rc;
}
