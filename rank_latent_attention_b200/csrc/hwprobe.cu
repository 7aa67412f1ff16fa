// Microbenchmarks of the sm_100a rates the FLARE++ kernels are designed
// around, one JSON line per measurement (run by rank_latent_attention_b200/
// hwprobe.py):
//   - MUFU ex2 throughput (fp32, packed f16x2, packed bf16x2) and the FMA
//     pipe's fp32 and packed f32x2 FMA throughput, in results per clock per SM;
//   - exp2_poly3 (the kernels' FMA-pipe exponential) in results per clock per SM;
//   - tcgen05.mma rate of back-to-back M=128 K=16 bf16 MMAs: N = 64 from one
//     thread of a divergent branch and from a whole warp under elect.sync;
//     N = 64, 128, 256 with A in shared memory (SS) and in TMEM (TS), in
//     clocks per MMA and MACs per clock;
//   - mbarrier wake-up latency: clocks from one warp's arrive to another
//     warp's try_wait (with a suspend-time hint) returning.
// Every wait is bounded; no TMA, no peer memory.
#include <cuda_runtime.h>
#include <stdio.h>

#include "common.cuh"

using namespace flare;

namespace {

constexpr int kRepsAlu = 4096;

// ------------------------------------------------------------------ pipes
// MODE 0: ex2.approx.ftz.f32; 1: ex2.approx.f16x2; 2: ex2.approx.ftz.bf16x2;
// 3: fma.rn.f32; 4: fma.rn.f32x2; 5: exp2_poly3_x2.  Eight independent chains
// per thread (each ex2 result negated, so that the chains stay finite); the
// clock count of CTA 0 is written to clk.  Launched with enough dynamic shared
// memory that only one CTA fits on an SM.
template <int MODE>
__global__ void __launch_bounds__(512) pipe_kernel(int reps, float* sink, long long* clk) {
  float a[8];
  uint32_t h[8];
  uint64_t p[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a[i] = -1.f - 1e-3f * (threadIdx.x + i);
    h[i] = 0x3c003c00u + i;  // small fp16 / bf16 pairs
    p[i] = ptx::f2(a[i], a[i] * 0.5f);
  }
  __syncthreads();
  const long long t0 = clock64();
  for (int r = 0; r < reps; ++r) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if constexpr (MODE == 0) {
        asm volatile("ex2.approx.ftz.f32 %0, %0;\n\tneg.f32 %0, %0;" : "+f"(a[i]));
      } else if constexpr (MODE == 1) {
        asm volatile("ex2.approx.f16x2 %0, %0;\n\tneg.f16x2 %0, %0;" : "+r"(h[i]));
      } else if constexpr (MODE == 2) {
        asm volatile("ex2.approx.ftz.bf16x2 %0, %0;\n\tneg.bf16x2 %0, %0;" : "+r"(h[i]));
      } else if constexpr (MODE == 3) {
        asm volatile("fma.rn.f32 %0, %0, 0f3F7FFFFF, 0fBF000000;" : "+f"(a[i]));
      } else if constexpr (MODE == 4) {
        p[i] = ptx::fma2(p[i], ptx::f2(0.99999994f, 0.99999994f), ptx::f2(-0.5f, -0.5f));
      } else {
        p[i] = exp2_poly3_x2(p[i]);
        p[i] = ptx::fma2(p[i], ptx::f2(-1.f, -1.f), ptx::f2(-0.5f, -0.5f));  // keep the input in range
      }
    }
  }
  __syncthreads();
  const long long t1 = clock64();
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float lo, hi;
    ptx::f2_split(p[i], lo, hi);
    acc += a[i] + __uint_as_float(h[i]) + lo + hi;
  }
  if (acc == 1234.5f) sink[threadIdx.x] = acc;  // never true; keeps the chains live
  if (threadIdx.x == 0 && blockIdx.x == 0) *clk = t1 - t0;
}

// ------------------------------------------------------------------ tcgen05.mma issue
// One CTA; warp 0 allocates 512 TMEM columns.  ELECT = false: thread 0 alone
// (a divergent branch) issues n MMAs; true: warp 1 runs the loop as a whole
// and issues each MMA under elect.sync.  M = 128, K = 16, N = NN.  The
// operands are zeros in shared memory in the 128-byte-swizzled K-major layout
// (A 128 x 64, B NN x 64 bf16); TS = true reads A from TMEM instead (columns
// [256, 264), zeroed first), the form the kernels' P.V products take.
template <bool ELECT, int NN, bool TS>
__global__ void __launch_bounds__(64) mma_issue_kernel(int n, long long* clk, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t taddr;
  using G = TileGeom<64>;
  static_assert(NN == 64 || NN == 128 || NN == 256, "N");
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (128 + NN) * 128 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  ptx::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(&taddr, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tm = taddr;
  constexpr uint32_t kColA = 256;
  if (TS) {
    // zero the A columns: warp w writes TMEM lanes [32 w, +32) (warps 0-1
    // reach lanes 0-63; the other lanes hold whatever was there, which only
    // changes the values, not the timing)
    const uint32_t z[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    ptx::tmem_st8(tm + (static_cast<uint32_t>(warp * 32) << 16) + kColA, z);
    ptx::tmem_wait_st();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t base = ptx::smem_u32(smem);
  const uint64_t dA = G::kmajor(base, 128, 0);
  const uint64_t dB = G::kmajor(base + 128 * 128, NN, 0);
  constexpr uint32_t kIdesc = ptx::idesc_bf16(128, NN, 0, 0);
  auto issue = [&](int i) {
    if (TS) {
      ptx::mma_ts(tm, tm + kColA, dB, kIdesc, i > 0 ? 1u : 0u);
    } else {
      ptx::mma_ss(tm, dA, dB, kIdesc, i > 0 ? 1u : 0u);
    }
  };
  long long t0 = 0, t1 = 0;
  if (!ELECT && threadIdx.x == 0) {
    t0 = clock64();
    for (int i = 0; i < n; ++i) issue(i);
    ptx::mma_commit(&bar);
    if (!ptx::mbar_wait_drain(&bar, 0)) atomicExch(status, 1);
    t1 = clock64();
  }
  if (ELECT && warp == 1) {
    t0 = clock64();
    for (int i = 0; i < n; ++i) {
      if (ptx::elect_one()) issue(i);
      __syncwarp();
    }
    if (ptx::elect_one()) ptx::mma_commit(&bar);
    __syncwarp();
    if (!ptx::mbar_wait_drain(&bar, 0)) atomicExch(status, 1);
    t1 = clock64();
    if (threadIdx.x != 32) t0 = t1 = 0;
  }
  if (t1 != 0) *clk = t1 - t0;
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tm, 512);
  }
}

template <bool ELECT, int NN, bool TS>
void mma_rate(int n, long long* clk, int* status) {
  const int smem = (128 + NN) * 128 + 1024;
  auto k = mma_issue_kernel<ELECT, NN, TS>;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return;
  long long c = 0;
  for (int it = 0; it < 2; ++it) k<<<1, 64, smem>>>(n, clk, status);
  if (cudaMemcpy(&c, clk, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess) c = -1;
  const double per = static_cast<double>(c) / n;
  printf("{\"probe\": \"tcgen05.mma M128 N%d K16 bf16 %s, back to back\", \"issuer\": \"%s\", \"mmas\": %d, "
         "\"clocks_per_mma\": %.1f, \"mac_per_clk\": %.0f}\n",
         NN, TS ? "TS (A in TMEM)" : "SS", ELECT ? "warp, elect.sync" : "one thread (divergent)", n, per,
         128.0 * NN * 16 / per);
}

// ------------------------------------------------------------------ mbarrier wake-up
// Warp 1 waits on a barrier phase with try_wait (suspend-time hint); warp 0
// arrives after a delay.  Per round: clock of the arrive and of the wake-up
// (both on this SM's clock).
__global__ void __launch_bounds__(64) mbar_wake_kernel(int rounds, long long* out, int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile long long t_arrive;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
  }
  __syncthreads();
  for (int r = 0; r < rounds; ++r) {
    if (threadIdx.x == 0) {
      const long long t = clock64();
      while (clock64() - t < 20000) {
      }
      t_arrive = clock64();
      ptx::mbar_arrive(&bar);
    }
    if (threadIdx.x == 32) {
      bool ok = ptx::mbar_try_wait(&bar, r & 1);
      const long long tw = clock64();
      for (int i = 0; !ok; ++i) {
        ok = ptx::mbar_try_wait_sleep(&bar, r & 1, 20000u);
        if (!ok && clock64() - tw > (1ll << 31)) break;
      }
      const long long t1 = clock64();
      if (!ok) atomicExch(status, 1);
      out[r] = t1 - t_arrive;
    }
    __syncthreads();
  }
}

constexpr int kOneCtaPerSmBytes = 150 * 1024;

template <int MODE>
double pipe_rate(const char* name, int results_per_instr, int sms, float* sink, long long* clk) {
  if (cudaFuncSetAttribute(pipe_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kOneCtaPerSmBytes) !=
      cudaSuccess)
    return -1;
  pipe_kernel<MODE><<<sms, 512, kOneCtaPerSmBytes>>>(kRepsAlu, sink, clk);  // warm
  pipe_kernel<MODE><<<sms, 512, kOneCtaPerSmBytes>>>(kRepsAlu, sink, clk);
  long long c = 0;
  if (cudaMemcpy(&c, clk, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess || c <= 0) return -1;
  const double instr = 512.0 * kRepsAlu * 8;  // warp-lane instructions per SM
  const double rate = instr * results_per_instr / static_cast<double>(c);
  printf("{\"probe\": \"%s\", \"results_per_clk_per_sm\": %.2f, \"clocks\": %lld}\n", name, rate, c);
  return rate;
}

}  // namespace

int main() {
  float* sink = nullptr;
  long long* clk = nullptr;
  int* status = nullptr;
  if (cudaMalloc(&sink, 512 * sizeof(float)) != cudaSuccess || cudaMalloc(&clk, 1024 * sizeof(long long)) != cudaSuccess ||
      cudaMalloc(&status, sizeof(int)) != cudaSuccess) {
    printf("{\"error\": \"cudaMalloc\"}\n");
    return 1;
  }
  cudaMemset(status, 0, sizeof(int));
  cudaDeviceProp prop;
  cudaGetDeviceProperties(&prop, 0);
  printf("{\"device\": \"%s\", \"sms\": %d, \"cc\": \"%d.%d\"}\n", prop.name, prop.multiProcessorCount, prop.major,
         prop.minor);
  pipe_rate<0>("ex2.approx.ftz.f32", 1, prop.multiProcessorCount, sink, clk);
  pipe_rate<1>("ex2.approx.f16x2", 2, prop.multiProcessorCount, sink, clk);
  pipe_rate<2>("ex2.approx.ftz.bf16x2", 2, prop.multiProcessorCount, sink, clk);
  pipe_rate<3>("fma.rn.f32", 1, prop.multiProcessorCount, sink, clk);
  pipe_rate<4>("fma.rn.f32x2", 2, prop.multiProcessorCount, sink, clk);
  // exp2_poly3_x2 plus one fma.rn.f32x2 that keeps its input in range
  pipe_rate<5>("exp2_poly3_x2 (+1 fma.f32x2)", 2, prop.multiProcessorCount, sink, clk);

  for (int n : {256, 1024}) {
    mma_rate<false, 64, false>(n, clk, status);
    mma_rate<true, 64, false>(n, clk, status);
  }
  mma_rate<true, 128, false>(1024, clk, status);
  mma_rate<true, 256, false>(1024, clk, status);
  mma_rate<true, 64, true>(1024, clk, status);
  mma_rate<true, 128, true>(1024, clk, status);
  mma_rate<true, 256, true>(1024, clk, status);

  const int rounds = 64;
  mbar_wake_kernel<<<1, 64>>>(rounds, clk, status);
  long long w[64];
  if (cudaMemcpy(w, clk, sizeof(w), cudaMemcpyDeviceToHost) == cudaSuccess) {
    long long lo = w[1], hi = w[1], sum = 0;
    for (int r = 1; r < rounds; ++r) {
      lo = w[r] < lo ? w[r] : lo;
      hi = w[r] > hi ? w[r] : hi;
      sum += w[r];
    }
    printf("{\"probe\": \"mbarrier arrive -> try_wait (suspend hint) returns\", \"clocks_mean\": %.0f, "
           "\"clocks_min\": %lld, \"clocks_max\": %lld}\n",
           static_cast<double>(sum) / (rounds - 1), lo, hi);
  }
  int st = 0;
  cudaMemcpy(&st, status, sizeof(int), cudaMemcpyDeviceToHost);
  const cudaError_t e = cudaDeviceSynchronize();
  printf("{\"status\": %d, \"cuda\": \"%s\"}\n", st, cudaGetErrorString(e));
  return (st == 0 && e == cudaSuccess) ? 0 : 1;
}
