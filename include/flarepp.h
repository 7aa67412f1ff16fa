/*
 * flarepp.h -- C ABI of the FLARE++ token-mixer forward pass for NVIDIA B200
 * (sm_100a).  Implemented by libflarepp.so (rank_latent_attention_b200/).
 *
 * The mixer routes N tokens through M << N latents, per head (b, h), in three
 * chained attention steps with scale s = 1:
 *
 *   seed encode     Q_dyn = softmax_N(Q~ K^T) V      Q~ = learned seeds of head h
 *   routing encode  Z     = softmax_N(Q_dyn K^T) V
 *   decode          Y     = softmax_M(K Q_dyn^T) Z
 *
 * Sources: the FLARE encode Z_h = SDPA(Q_h, K_h, V_h, s=1) and decode
 * Y_h = SDPA(K_h, Q_h, Z_h, s=1) ("FLARE: Fast Low-rank Attention Routing
 * Engine", review page, section "Основной механизм FLARE"); FLARE++ replaces
 * the learned queries by Q_dyn, produced by one extra encode driven by the
 * seeds ("FLARE++: Low-rank attention with dynamic attention routing",
 * section "Méthodologie : FLARE++", items "Synthèse de Requêtes Dynamiques"
 * and "Routage Encode-Décode"; abstract).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Tensors are dense, row-major, contiguous, in DEVICE memory owned by the
 *   caller, and 16-byte aligned:
 *     seeds / fixed queries  [H][M][D]      (shared by the batch)
 *     batched queries        [B][H][M][D]
 *     K, V, Y                [B][H][N][D]
 *     Q_dyn, Z               [B][H][M][D]
 * - dtype is FLARE_BF16 (bf16 storage, fp32 accumulation and fp32 softmax on
 *   the tensor cores; intermediates Q_dyn and Z are stored as bf16, rounded to
 *   nearest, as three chained bf16 SDPA calls would return them) or FLARE_F32
 *   (fp32 everywhere, CUDA-core path); every tensor of a call has that dtype.
 *   FLARE_BF16_F32OUT (flarepp_mix / flarepp_mix_debug / flarepp_mix_host
 *   only) takes bf16 seeds, K and V and returns Q_dyn, Z and Y in fp32: for
 *   inputs whose outputs are so heavy-tailed (or whose logits are so large)
 *   that bf16 storage of the chain exceeds an accuracy budget.  For
 *   M % 16 == 0 and D <= 64 it runs on the tensor cores in split precision:
 *   the rounded MMA operands are carried as pairs hi = round(x),
 *   lo = round(x - hi) of 16-bit numbers and each product takes one MMA per
 *   part (the encodes' softmax weights and Q_dyn as bf16 pairs, Z as an fp16
 *   pair scaled per head by a power of two; the decode's weights, in [0, 1],
 *   as fp16).  Other sizes run on the fp32 CUDA-core kernels.
 * - Supported sizes: B >= 1, H >= 1, B*H <= 65535, 1 <= N < 2^31 - 256,
 *   D in {16, 32, 64, 128}, 1 <= M <= 256; for FLARE_BF16 additionally
 *   M % 16 == 0.  N needs no alignment: the last tile of each head is masked.
 * - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Work is enqueued asynchronously; nothing synchronises the host.
 * - Return value: a flare_status_t.  Invalid arguments (null or unaligned
 *   pointers, host pointers, unsupported sizes, a workspace that is too
 *   small) return an error before any work is enqueued.  FLARE_ERR_CUDA means
 *   a launch failed; the CUDA error is left for cudaGetLastError.  The kernels
 *   never trap: a wait inside a kernel that exceeds the wait limit records
 *   FLARE_ERR_TIMEOUT in a per-device status word that flare_check_status
 *   reports.
 * - Workspace: device scratch of at least the size returned by the matching
 *   *_workspace_size function, owned by the caller, 256-byte aligned.  If
 *   workspace is NULL the library allocates it with cudaMallocAsync on the
 *   stream and frees it with cudaFreeAsync after the last kernel.
 */
#ifndef FLAREPP_H
#define FLAREPP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLARE_F32 = 0,         /* fp32 storage and arithmetic (CUDA cores)                            */
  FLARE_BF16 = 1,        /* bf16 storage; tcgen05 bf16 MMAs, fp32 accumulation and softmax      */
  FLARE_BF16_F32OUT = 2  /* mixer only: bf16 seeds/K/V; split-precision MMAs, fp32 Q_dyn, Z, Y   */
} flare_dtype_t;

typedef enum {
  FLARE_OK = 0,
  FLARE_ERR_INVALID_ARG = 1,  /* null/unaligned/host pointer, bad enum, workspace too small */
  FLARE_ERR_UNSUPPORTED = 2,  /* sizes outside the supported set */
  FLARE_ERR_CUDA = 3,         /* a CUDA call or kernel launch failed */
  FLARE_ERR_TIMEOUT = 4       /* a kernel gave up waiting (reported by flare_check_status) */
} flare_status_t;

/* Bytes of workspace flare_encode needs for these sizes (0 for invalid sizes). */
size_t flare_encode_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);

/* Bytes of workspace flarepp_mix / flarepp_mix_debug need (0 for invalid sizes). */
size_t flarepp_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);

/*
 * FLARE encode: Z[b,h] = softmax_N(Q K[b,h]^T) V[b,h], softmax over the N tokens.
 * ("FLARE" review page, "Основной механизм FLARE", encode step.)
 *   Q          [H][M][D] if q_batched == 0 (learned queries, shared by the batch)
 *              [B][H][M][D] if q_batched == 1
 *   K, V       [B][H][N][D]
 *   Z          [B][H][M][D] output
 * The token axis is split across CTAs; the per-split softmax statistics are
 * merged exactly (log-sum-exp) in a second kernel.  With one CTA per head
 * (flare_encode_splits() == 1, tensor-core modes) the encode writes the
 * normalised result itself and no second kernel runs.
 */
int flare_encode(const void* Q, int q_batched, const void* K, const void* V, void* Z, int B, int H, int64_t N,
                 int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * FLARE decode: Y[b,h][n] = softmax_M(K[b,h][n] . Q^T) Z[b,h], softmax over the
 * M latents, one row per token.  ("FLARE" review page, "Основной механизм
 * FLARE", decode step Y = SDPA(K, Q, Z, s=1).)
 *   K          [B][H][N][D]
 *   Q          latent keys: [H][M][D] if q_batched == 0, [B][H][M][D] if 1
 *   Z          [B][H][M][D]
 *   Y          [B][H][N][D] output
 * Needs no workspace.
 */
int flare_decode(const void* K, const void* Q, int q_batched, const void* Z, void* Y, int B, int H, int64_t N,
                 int M, int D, int dtype, void* stream);

/*
 * Token-sharded (context-parallel) encode, in two calls.  The FLARE++ page
 * ("FLARE++: Low-rank attention with dynamic attention routing", section
 * "Contributions Clés", multi-GPU context-parallelism item) shards the input
 * tokens over devices and exchanges only the latent outputs and the softmax
 * statistics, never the tokens.  With shard r's logits s_mn = Q_m . K_n over
 * its tokens n in r:
 *   O_r[m]   = sum_{n in r} exp(s_mn) V_n / sum_{n in r} exp(s_mn)
 *   lse_r[m] = ln sum_{n in r} exp(s_mn)
 * and the encode over the union of the shards is exactly
 *   out[m] = sum_r exp(lse_r[m] - L[m]) O_r[m],   L[m] = ln sum_r exp(lse_r[m]).
 *
 * flare_encode_lse: one shard's (O_r, lse_r).
 *   Q          [H][M][D] (q_batched 0) or [B][H][M][D] (q_batched 1), dtype
 *   K, V       [B][H][N][D] this shard's tokens, dtype; may be NULL when N == 0
 *   O          [B][H][M][D] fp32 output, whatever dtype is
 *   lse        [B][H][M] fp32 output (natural log); needs 4-byte alignment only
 *   N          the shard's token count, N >= 0.  N == 0 (an empty shard)
 *              writes O = 0 and lse = -inf, which carry no weight when combined.
 * dtype FLARE_BF16 or FLARE_F32 (the inputs' type and the arithmetic as in
 * flare_encode); workspace as flare_encode (flare_encode_lse_workspace_size;
 * 0 bytes for N == 0).
 *
 * flare_lse_combine: the exact combination of R shards' results.
 *   O_parts    R arrays [B][H][M][D] fp32 (one flare_encode_lse output per
 *              shard, in any order: it changes only the rounding)
 *   lse_parts  R arrays [B][H][M] fp32 (4-byte alignment)
 *   part_stride  floats from shard r's arrays to shard r+1's, the same for
 *              O_parts and lse_parts; 0 = dense stacks [R][B][H][M][D] and
 *              [R][B][H][M].  With one buffer of R rows [O_r | lse_r] (what
 *              one all-gather of each device's [O | lse] returns), pass
 *              O_parts = buf, lse_parts = buf + B*H*M*D and
 *              part_stride = B*H*M*(D+1).
 *   out        [B][H][M][D] output, dtype (FLARE_BF16: rounded to nearest)
 *   lse_out    [B][H][M] fp32 output L, or NULL
 * A latent whose shards are all empty gets out = 0 and L = -inf.  One kernel;
 * no workspace.  Sizes as flare_encode with N = 1.
 */
size_t flare_encode_lse_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);

/*
 * FLARE++ mixer backward: the gradients of L = sum(dY * Y) with respect to
 * the seeds, K and V, where Y = flarepp_mix(seeds, K, V).  The pages train
 * the mixer end to end ("FLARE++: Low-rank attention with dynamic attention
 * routing", "Méthodologie : FLARE++": the routing is SDPA calls alone);
 * this is the chain rule through the three steps:
 *   decode   dZ = P3^T dY,  dS3 = P3 (dY Z^T - rowsum(dY * Y))
 *   routing  dS2 = A2 (dZ V^T - rowsum(dZ * Z)),
 *            dQ_dyn = dS3^T K + dS2 K
 *   seed     dS1 = A1 (dQ_dyn V^T - rowsum(dQ_dyn * Q_dyn))
 *   d_seeds = sum_b dS1 K,  dK = (dS3 + dS2^T) Q_dyn + dS1^T seeds,
 *   dV = A2^T dZ + A1^T dQ_dyn
 * with A1, A2 the encode weights (softmax over tokens) and P3 the decode
 * weights (softmax over latents).
 *   seeds      [H][M][D]            K, V, dY   [B][H][N][D]
 *   d_seeds    [H][M][D] output (summed over the batch, which shares the seeds)
 *   dK, dV     [B][H][N][D] outputs
 * The call recomputes the two encodes (Q_dyn and Z exactly as flarepp_mix
 * stores them, bf16 on FLARE_BF16, with their log-sum-exps) and then runs
 * eight kernels: on FLARE_BF16 with D <= 64 the five token/latent passes are
 * tcgen05 tensor-core kernels (bf16 operands, fp32 accumulation), otherwise
 * fp32 CUDA-core kernels; the three partial-sum reductions are fp32.  Stored values such as Q_dyn and Z are used
 * as stored, so the result is the gradient of the computed chain with each
 * rounding taken as the identity.  Everything after the loads is fp32; dK, dV
 * and d_seeds are stored in dtype.  dtype FLARE_BF16 or FLARE_F32; the
 * workspace comes from flarepp_mix_backward_workspace_size.
 */
size_t flarepp_mix_backward_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);

/*
 * Forward and backward with saved state, as a training step runs them:
 * flarepp_mix_save is flarepp_mix that also keeps what the backward needs,
 * and flarepp_mix_backward_saved is flarepp_mix_backward without its two
 * recomputed encodes (it reads that state instead).
 *   saved      device buffer of flarepp_saved_bytes(B, H, M, D, dtype) bytes,
 *              256-byte aligned, owned by the caller; holds, each region
 *              256-byte aligned: Q_dyn and Z [B][H][M][D] (dtype) as the
 *              forward stored them, then lse1 and lse2 [B][H][M] fp32 (the
 *              seed and routing encodes' log-sum-exps, natural log).
 * The gradients equal flarepp_mix_backward's bit for bit when the forward
 * ran on the same inputs.  dtype FLARE_BF16 or FLARE_F32; workspaces as
 * flarepp_mix and flarepp_mix_backward.
 */
size_t flarepp_saved_bytes(int B, int H, int M, int D, int dtype);

/*
 * Token-sharded backward (training with the tokens of one cloud spread over
 * ranks, as in the FLARE++ page's context-parallel item, "Contributions
 * Clés").  Each rank holds its tokens' K, V, dY and the replicated state of
 * the sharded forward (`saved`: Q_dyn, Z, lse1, lse2 of the whole cloud, as
 * flarepp_mix_save lays them out).  The backward's token reductions (dZ,
 * dQ_dyn, d_seeds) need every rank's tokens, so it runs in four phases;
 * between phases the caller sums `exchange` over the ranks (an all-reduce):
 *   phase 0: statistics and the decode pass; exchange = [dZ | dQ_dyn decode
 *            part], 2 x [B][H][M][D] fp32
 *   phase 1: routing pass; exchange = dQ_dyn routing part, [B][H][M][D]
 *   phase 2: seed pass; exchange = d_seeds, [H][M][D] fp32
 *   phase 3: d_seeds (dtype, the summed value) and this rank's dK, dV
 * N is this rank's token count (0 allowed: the rank contributes zeros).
 * The workspace (flarepp_backward_shard_workspace_size bytes) must be the
 * same buffer in all four calls and is required; exchange holds at least
 * flarepp_backward_shard_exchange_floats floats.  With one rank and no
 * exchange between phases the result equals flarepp_mix_backward_saved's
 * bit for bit.
 */
size_t flarepp_backward_shard_exchange_floats(int B, int H, int M, int D);
size_t flarepp_backward_shard_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);
int flarepp_mix_backward_shard(int phase, const void* seeds, const void* K, const void* V, const void* dY,
                               const void* saved, float* exchange, void* d_seeds, void* dK, void* dV, int B, int H,
                               int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes,
                               void* stream);
int flarepp_mix_save(const void* seeds, const void* K, const void* V, void* Y, void* saved, int B, int H, int64_t N,
                     int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream);
int flarepp_mix_backward_saved(const void* seeds, const void* K, const void* V, const void* dY, const void* saved,
                               void* d_seeds, void* dK, void* dV, int B, int H, int64_t N, int M, int D, int dtype,
                               void* workspace, size_t workspace_bytes, void* stream);
int flarepp_mix_backward(const void* seeds, const void* K, const void* V, const void* dY, void* d_seeds, void* dK,
                         void* dV, int B, int H, int64_t N, int M, int D, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream);
int flare_encode_lse(const void* Q, int q_batched, const void* K, const void* V, float* O, float* lse, int B,
                     int H, int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes,
                     void* stream);
int flare_lse_combine(const float* O_parts, const float* lse_parts, int R, int64_t part_stride, void* out,
                      float* lse_out, int B, int H, int M, int D, int dtype, void* stream);

/*
 * FLARE++ mixer forward: seed encode -> routing encode -> decode (see top).
 *   seeds      [H][M][D]
 *   K, V       [B][H][N][D]
 *   Y          [B][H][N][D] output (fp32 when dtype is FLARE_BF16_F32OUT)
 * K and V are streamed from memory three times in all (K, V; K, V; K) and Y
 * written once; Q_dyn and Z live in the workspace.
 */
int flarepp_mix(const void* seeds, const void* K, const void* V, void* Y, int B, int H, int64_t N, int M, int D,
                int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Same as flarepp_mix, and also returns the intermediates: Q_dyn and Z
 * ([B][H][M][D], dtype) are written to the caller's buffers, which the later
 * steps then read, so the returned values are exactly the ones used.
 */
int flarepp_mix_debug(const void* seeds, const void* K, const void* V, void* Y, void* Q_dyn, void* Z, int B, int H,
                      int64_t N, int M, int D, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * flarepp_mix_host: flarepp_mix with seeds, K, V and Y in HOST memory (same
 * layouts and dtypes; page-locked memory lets the copies run asynchronously,
 * pageable memory works but its copies stage through the driver).  The
 * (b, h) heads are independent ("FLARE++" page, "Méthodologie : FLARE++":
 * each head routes only its own tokens), so the call streams them through the
 * GPU one head at a time: the copy of head c + 1 in, the mix of head c and the
 * copy of head c - 1 out overlap on two library-owned copy streams and the
 * caller's stream, using both directions of the host link at once.  Returns
 * once everything is enqueued; when `stream` has completed, Y holds the
 * result.  workspace: device memory of at least
 * flarepp_mix_host_workspace_size() bytes (two heads' K, V and Y, the seeds
 * and one head's mix workspace), or NULL to allocate on `stream`.  Calls are
 * serialised within a process while they enqueue.  Errors as for flarepp_mix;
 * a device pointer where host memory is expected is FLARE_ERR_INVALID_ARG.
 */
size_t flarepp_mix_host_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);
int flarepp_mix_host(const void* seeds, const void* K, const void* V, void* Y, int B, int H, int64_t N, int M, int D,
                     int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word.  Returns FLARE_OK or the first error a kernel recorded since the last
 * check (FLARE_ERR_TIMEOUT); *site (if not NULL) receives the kernel role
 * that recorded it (1-3 encode producer/MMA/softmax, 4-6 decode producer/
 * MMA/softmax, 7-12 the backward's tensor-core kernels, 13 the wait
 * self-test).  Returns
 * FLARE_ERR_CUDA if the synchronisation itself fails.
 */
int flare_check_status(void* stream, int* site);

/*
 * Self-test of the kernels' bounded waits: one warp waits on an mbarrier
 * that nothing arrives at.  The wait gives up after limit_ms (1..1000) of
 * %globaltimer, the kernel records FLARE_ERR_TIMEOUT with site 13 in the
 * status word (as any kernel that gives up waiting does) and returns; the
 * context stays usable.  flare_check_status then returns FLARE_ERR_TIMEOUT.
 * The probe holds no TMA copy, MMA or tensor memory.
 */
int flare_selftest_wait_timeout(int limit_ms, void* stream);

/* Static, human-readable name of a status code. */
const char* flare_status_string(int status);

/* Number of kernels the last successful call on this host thread enqueued. */
int flare_last_launch_count(void);

/*
 * Name of the CUDA error the library's own CUDA runtime last recorded on this
 * host thread ("no error" if none), without clearing it: after a call returned
 * FLARE_ERR_CUDA this names the failed launch or CUDA call.  The library links
 * its CUDA runtime statically, so the caller's cudaGetLastError does not see
 * that state.  Static string.
 */
const char* flare_cuda_error_string(void);

/*
 * Tuning / test hooks (process-wide, not thread-safe against concurrent calls):
 *   flare_set_split_override(s): use s CTAs per head along the tokens in
 *     every token-split kernel, each clamped to that kernel's number of token
 *     tiles (64 tokens for the encode and the backward's latent-side kernel,
 *     128 for the decode, the statistics and the token-gradient kernels); 0
 *     restores the built-in choice: the count that minimises (waves of the
 *     SMs' resident CTA slots) x (tiles per CTA + a fixed per-CTA cost of
 *     384 tokens), among counts that keep a CTA at most ~32k tokens.
 *   flare_set_wait_limit_ms(ms): how long a tensor-core kernel waits on one
 *     barrier before recording FLARE_ERR_TIMEOUT and returning (default 2000).
 *   flare_set_launch_overlap(mode): whether the mixer's merges, routing
 *     encode and decode are launched with programmatic stream serialisation,
 *     so that each may start its set-up (barriers, tensor memory, the first
 *     K/V loads) while the kernel before it finishes; every such kernel
 *     waits for its predecessor before it reads that kernel's output, and the
 *     seed encode never overlaps whatever precedes the call.  1 always, 0
 *     never, -1 (the default) when each encode CTA has at most 64 token
 *     tiles, where the fixed cost of a launch is a large share of the call.
 * All return the previous value.
 */
int flare_set_split_override(int splits);
/*
 * The number of CTAs per head along the tokens that the tensor-core encode
 * uses for B x H heads of N tokens (the built-in choice, or the override):
 * with 1, the encode writes its normalised result and log-sum-exp itself
 * and no lse_merge_kernel follows it.  0 for B, H or N below 1.  Reads
 * only host state; no device work.
 */
int flare_encode_splits(int B, int H, int64_t N);
int flare_set_wait_limit_ms(int ms);
int flare_set_launch_overlap(int mode);

/*
 * Communication matrix of the latent routing, per head (b, h):
 *   C = W_enc W_dec   (M x M),  W_enc = softmax_N(Q K^T) (M x N, over tokens),
 *                                W_dec = softmax_M(K Q^T) (N x M, over latents),
 * scale 1.  The token-to-token matrix W = W_dec W_enc (N x N, "FLARE: Fast
 * Low-rank Attention Routing Engine" review page, section "Матрица
 * коммуникации низкого ранга") has rank at most M, and its nonzero
 * eigenvalues are those of C (same page, section "Спектральный анализ": the
 * spectrum in O(M^3 + M^2 N)); C is row-stochastic, so its leading
 * eigenvalue is 1.  For FLARE++ pass the routing queries Q_dyn as Q
 * (q_batched = 1).
 *
 * Q: [H][M][D] (q_batched = 0) or [B][H][M][D]; K: [B][H][N][D]; C:
 * [B][H][M][M].  dtype: FLARE_F32 (fp32 throughout on CUDA cores, C fp32);
 * FLARE_BF16 (bf16 Q and K, C bf16); FLARE_BF16_F32OUT (bf16 Q and K, C
 * fp32).  All pointers are device memory owned by the caller, 16-byte
 * aligned.  The library forms C only: the O(M^3) eigen-solve of the M x M
 * matrices is left to the caller.
 * bf16 inputs with M % 16 == 0 and D <= 64 take one pass over the tokens on
 * the tensor cores: both weights are functions of the same logits,
 * W_enc[m][n] = exp(s_nm - L2_m) and W_dec[n][m] = exp(s_nm - L3_n), so with
 * the per-latent log-sum-exp L2 (an encode's merge) C is a plain sum over
 * tokens of W_enc[:, n] W_dec[n, :], accumulated in fp32 from fp16 weights
 * (both lie in [0, 1]; 4 launches: encode, merge, the C kernel, the sum of its token-split
 * partials).  Other sizes (and FLARE_F32) use the library's decode and
 * encode: ceil(M / D) rounds of a decode with Z = D columns of the M x M
 * identity (giving those columns of W_dec) and an encode with that block as
 * V; FLARE_BF16_F32OUT is then FLARE_ERR_UNSUPPORTED.  workspace: at least
 * flare_communication_workspace_size() bytes, or NULL to allocate on the
 * stream.  Errors as for flare_encode.
 */
size_t flare_communication_workspace_size(int B, int H, int64_t N, int M, int D, int dtype);
int flare_communication_matrix(const void* Q, int q_batched, const void* K, void* C, int B, int H, int64_t N, int M,
                               int D, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/* Kernel kinds reported by the launch profiler. */
typedef enum {
  FLARE_KERNEL_ENCODE_TC = 1,   /* split-token tcgen05 encode (partials) */
  FLARE_KERNEL_MERGE = 2,       /* log-sum-exp merge of encode partials  */
  FLARE_KERNEL_DECODE_TC = 3,   /* tcgen05 decode                        */
  FLARE_KERNEL_ENCODE_F32 = 4,  /* fp32 CUDA-core encode (partials)      */
  FLARE_KERNEL_DECODE_F32 = 5,       /* fp32 CUDA-core decode                 */
  FLARE_KERNEL_BWD_TOKEN_STATS = 6,  /* backward: per-token lse3, delta       */
  FLARE_KERNEL_BWD_LATENT = 7,       /* backward: latent-side partials        */
  FLARE_KERNEL_BWD_REDUCE = 8,       /* backward: sums of those partials      */
  FLARE_KERNEL_BWD_TOKEN_GRAD = 9,   /* backward: dK, dV                      */
  FLARE_KERNEL_COMM_TC = 10,         /* communication matrix, one pass        */
  FLARE_KERNEL_COMM_REDUCE = 11      /* sum of its token-split partials       */
} flare_kernel_kind_t;

/*
 * Launch profiler.  flare_profile_begin(n) makes the next n kernel launches
 * (of any call, on any stream) record a CUDA event just before and just after
 * the launch on the launching stream; nothing else changes and nothing
 * synchronises.  flare_profile_end synchronises on those events, writes up to
 * max_records durations (ms) and kernel kinds in launch order, releases the
 * events and returns the number of records written (negative status on
 * error).  Used by bench.py to time each kernel inside a timed region.
 */
int flare_profile_begin(int max_launches);
int flare_profile_end(float* ms, int* kinds, int max_records);

/*
 * flare_encode_noalloc: the FLARE encode of flare_encode (same arguments,
 * same kernels, same results) for callers that are not allowed to allocate
 * device memory.  Some code cannot call cudaMalloc or ask its caller for a
 * workspace: a library layer whose host framework already owns every byte of
 * the GPU through its own pool, a latency-critical loop where an allocation
 * (which may synchronise the device or fail under memory pressure) is not
 * acceptable, or a plug-in whose interface passes only inputs and outputs.
 * The pages have no counterpart to this entry point; it exists for such
 * callers only.
 *
 * The split-token softmax partials live in one scratch array of
 * FLARE_NOALLOC_SCRATCH_BYTES bytes that is part of the library itself, so
 * every GPU the library is loaded on holds that much memory until the
 * process exits.  The first call on each device looks up that array's
 * device address (with that device current), so make the first call on a
 * device before starting any stream capture.  Calls whose partials need more
 * than FLARE_NOALLOC_SCRATCH_BYTES (see flare_encode_workspace_size) return
 * FLARE_ERR_UNSUPPORTED before enqueuing anything; use flare_encode with a
 * workspace for those.  Nothing in the array has to start at zero: each call
 * writes every partial it later reads.  All calls share the one array, so
 * two calls whose kernels can overlap on the GPU (different streams without
 * ordering, or several host threads) race on it; order them on one stream.
 * dtype FLARE_F32 or FLARE_BF16.  No cudaMalloc, cudaFree or other
 * allocating call is made.
 */
#define FLARE_NOALLOC_SCRATCH_BYTES (16u << 20)
int flare_encode_noalloc(const void* Q, int q_batched, const void* K, const void* V, void* Z, int B, int H,
                         int64_t N, int M, int D, int dtype, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FLAREPP_H */
