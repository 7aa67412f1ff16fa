"""fp64 CPU oracle for the FLARE++ mixer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The library's CUDA path never calls it
and shares no code with it.

What it computes, per head (b, h), in float64, with scale s = 1 throughout:

1. seed encode      Q_dyn = softmax_N(Q~ K^T) V       (softmax over the N tokens)
2. routing encode   Z     = softmax_N(Q_dyn K^T) V
3. decode           Y     = softmax_M(K Q_dyn^T) Z    (softmax over the M latents)

Sources (page title, section):

* "FLARE: Fast Low-rank Attention Routing Engine" (review page), section
  "Основной механизм FLARE": the encode step Z_h = SDPA(Q_h, K_h, V_h, s=1)
  with Q_h in R^{MxD} and K_h, V_h in R^{NxD}; the decode step
  Y_h = SDPA(K_h, Q_h, Z_h, s=1).
* same page, section "Матрица коммуникации низкого ранга": the weights
  W_encode = softmax(Q K^T) (MxN, normalised over tokens),
  W_decode = softmax(K Q^T) (NxM, normalised over latents) and
  Y = (W_decode W_encode) V with W of rank at most M.
* "FLARE++: Low-rank attention with dynamic attention routing", section
  "Contributions Clés", multi-GPU context-parallelism item: the tokens are
  sharded over devices, each device encodes its own shard, and only the
  latent outputs and the softmax statistics cross devices
  (``encode_shard`` / ``combine_shards``).
* same page, section
  "Méthodologie : FLARE++": learned seeds Q~_h drive one extra encode call
  whose M outputs become the routing queries Q_h(X) (dynamic query
  synthesis), which then replace the learned queries in FLARE's encode-decode
  pair (routing encode-decode).  The abstract states the same: one extra
  encode call over the same N tokens.

Readings taken where the pages are silent (listed with the others in the
design notes): s = 1 in all three steps; the seed encode uses the same K and V
as the routing encode; Q_dyn is used as-is (no normalisation) both as the
routing queries and as the decode keys; softmax is max-subtracted, which is
the same function.

The backward (``flarepp_head_backward``) is the chain rule through the same
three steps, written out step by step; the pages train the mixer end to end
("FLARE++" page, "Méthodologie : FLARE++": the routing is built from SDPA
calls alone, so it is differentiable like any attention).

Every function here is "pinned" by tests in ``tests/test_oracle.py`` against
things other than itself: the hand-derived worked examples in
``tests/golden/``, a pure-Python brute force, torch's float64 SDPA, the dense
NxN communication matrix, its rank and spectrum, and invariants of the
definition.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "softmax",
    "sdpa",
    "attention_weights",
    "flare_encode",
    "flare_decode",
    "flarepp_head",
    "flarepp_mix",
    "flarepp_decode_rows",
    "communication_matrix",
    "communication_eigenvalues",
    "encode_shard",
    "combine_shards",
    "flarepp_head_backward",
    "flarepp_backward",
]


def softmax(S: np.ndarray, axis: int = -1) -> np.ndarray:
    """Max-subtracted softmax along ``axis`` in float64."""
    S = np.asarray(S, dtype=np.float64)
    E = np.exp(S - S.max(axis=axis, keepdims=True))
    return E / E.sum(axis=axis, keepdims=True)


def attention_weights(q: np.ndarray, k: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """softmax(scale * q k^T) normalised over the rows of k (the keys)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    return softmax(scale * (q @ k.T), axis=-1)


def sdpa(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float = 1.0) -> np.ndarray:
    """Scaled dot-product attention softmax(scale q k^T) v, one head, float64."""
    return attention_weights(q, k, scale) @ np.asarray(v, dtype=np.float64)


def flare_encode(Q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """FLARE encode of one head: the M queries gather the N tokens.

    ``FLARE`` review page, "Основной механизм FLARE", encode step:
    Z = SDPA(Q, K, V, s=1); Q is MxD, K and V are NxD, result MxD.
    """
    return sdpa(Q, K, V, 1.0)


def flare_decode(K: np.ndarray, Q: np.ndarray, Z: np.ndarray) -> np.ndarray:
    """FLARE decode of one head: each token's key queries the M latents.

    ``FLARE`` review page, "Основной механизм FLARE", decode step:
    Y = SDPA(K, Q, Z, s=1); the softmax runs over the M latents; result NxD.
    """
    return sdpa(K, Q, Z, 1.0)


def flarepp_head(seeds: np.ndarray, K: np.ndarray, V: np.ndarray):
    """The three chained steps of one FLARE++ head; returns (Q_dyn, Z, Y).

    ``FLARE++`` page, "Méthodologie : FLARE++": dynamic query synthesis
    (seeds query one extra encode over the tokens) followed by the standard
    encode-decode pair driven by the synthesised queries.
    """
    Q_dyn = flare_encode(seeds, K, V)
    Z = flare_encode(Q_dyn, K, V)
    Y = flare_decode(K, Q_dyn, Z)
    return Q_dyn, Z, Y


def flarepp_decode_rows(K: np.ndarray, Q_dyn: np.ndarray, Z: np.ndarray, rows) -> np.ndarray:
    """Decode output for the selected token rows only (each row is independent)."""
    K = np.asarray(K, dtype=np.float64)
    return flare_decode(K[np.asarray(rows)], Q_dyn, Z)


def flarepp_mix(seeds: np.ndarray, K: np.ndarray, V: np.ndarray, heads=None):
    """Whole mixer: seeds [H,M,D], K and V [B,H,N,D] -> (Q_dyn, Z, Y) float64.

    ``heads`` optionally restricts the work to a list of (b, h) pairs; the
    other entries of the outputs are left as NaN.
    """
    B, H, N, D = K.shape
    M = seeds.shape[1]
    Q_dyn = np.full((B, H, M, D), np.nan)
    Z = np.full((B, H, M, D), np.nan)
    Y = np.full((B, H, N, D), np.nan)
    todo = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    for b, h in todo:
        Q_dyn[b, h], Z[b, h], Y[b, h] = flarepp_head(seeds[h], K[b, h], V[b, h])
    return Q_dyn, Z, Y


def communication_matrix(Q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """The NxN global communication matrix W = W_decode W_encode of one head.

    ``FLARE`` review page, "Матрица коммуникации низкого ранга": W_encode =
    softmax(Q K^T) (MxN, over tokens), W_decode = softmax(K Q^T) (NxM, over
    latents); the decode output equals W V and W has rank at most M.
    """
    W_enc = attention_weights(Q, K)  # M x N
    W_dec = attention_weights(K, Q)  # N x M
    return W_dec @ W_enc


def communication_eigenvalues(Q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """Eigenvalues of W through the MxM product W_encode W_decode.

    ``FLARE`` review page, "Спектральный анализ": the spectrum of the learned
    communication matrices is obtained in O(M^3 + M^2 N) time.  The plainest
    reading: the nonzero eigenvalues of W_dec W_enc (NxN) are those of
    W_enc W_dec (MxM), which costs O(M^2 N) to form and O(M^3) to solve.
    Returned sorted by decreasing modulus.
    """
    W_enc = attention_weights(Q, K)
    W_dec = attention_weights(K, Q)
    ev = np.linalg.eigvals(W_enc @ W_dec)
    return ev[np.argsort(-np.abs(ev))]


def encode_shard(Q: np.ndarray, K: np.ndarray, V: np.ndarray):
    """One token shard's encode: (O, lse), O MxD, lse length M.

    ``FLARE++`` page, "Contributions Clés", multi-GPU context parallelism:
    a device holds only its shard of the tokens and sends out only latent
    outputs and softmax statistics.  With the shard's logits s_mn = Q_m . K_n:
    O[m] = softmax over the shard's tokens of s_m., applied to V (the
    shard-local encode) and lse[m] = log sum_n exp(s_mn).  A shard without
    tokens has O = 0 and lse = -inf.
    """
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    M, D = Q.shape[0], V.shape[1]
    if K.shape[0] == 0:
        return np.zeros((M, D)), np.full(M, -np.inf)
    S = Q @ K.T
    top = S.max(axis=1, keepdims=True)
    E = np.exp(S - top)
    tot = E.sum(axis=1)
    return (E @ V) / tot[:, None], top[:, 0] + np.log(tot)


def combine_shards(O_parts, lse_parts):
    """The encode over the union of disjoint token shards from their (O, lse).

    Token n of shard r has full-softmax weight exp(s_mn - L_m) =
    exp(s_mn - lse_r[m]) * exp(lse_r[m] - L_m), with L = log sum_r exp(lse_r),
    so out[m] = sum_r exp(lse_r[m] - L_m) O_r[m].  Returns (out, L); latents
    whose shards are all empty get out = 0 and L = -inf.
    """
    lse = np.stack([np.asarray(x, dtype=np.float64) for x in lse_parts])  # R x M
    O = np.stack([np.asarray(x, dtype=np.float64) for x in O_parts])  # R x M x D
    top = lse.max(axis=0)
    live = np.isfinite(top)
    w = np.zeros_like(lse)
    w[:, live] = np.exp(lse[:, live] - top[live])
    tot = w.sum(axis=0)
    out = np.zeros(O.shape[1:])
    out[live] = np.einsum("rm,rmd->md", w[:, live], O[:, live]) / tot[live, None]
    L = np.full(top.shape, -np.inf)
    L[live] = top[live] + np.log(tot[live])
    return out, L


def _softmax_backward(A: np.ndarray, dA: np.ndarray, c: np.ndarray) -> np.ndarray:
    """dS for rows A = softmax(S) given dA = dL/dA and each row's c = sum(A * dA)."""
    return A * (dA - c[:, None])


def flarepp_head_backward(seeds, K, V, dY, Q_dyn=None, Z=None):
    """Gradients of L = sum(dY * Y) for one FLARE++ head: (d_seeds, dK, dV).

    Forward (``flarepp_head``): S1 = Q~ K^T, A1 = softmax over tokens,
    Q_dyn = A1 V; S2 = Q_dyn K^T, A2 = softmax over tokens, Z = A2 V;
    S3 = K Q_dyn^T, P3 = softmax over latents, Y = P3 Z.  Backward, last step
    first:

      decode   dZ = P3^T dY;  dP3 = dY Z^T;  dS3 = P3 (dP3 - rowsum(dY * Y))
               dK += dS3 Q_dyn;  dQ_dyn += dS3^T K
      routing  dV += A2^T dZ;  dA2 = dZ V^T;  dS2 = A2 (dA2 - rowsum(dZ * Z))
               dQ_dyn += dS2 K;  dK += dS2^T Q_dyn
      seed     dV += A1^T dQ_dyn;  dA1 = dQ_dyn V^T;
               dS1 = A1 (dA1 - rowsum(dQ_dyn * Q_dyn))
               d_seeds = dS1 K;  dK += dS1^T Q~

    Each rowsum(dO * O) is the softmax backward's sum(A * dA) written with
    the step's output O = A X.  With Q_dyn / Z given (as a reduced-precision
    forward stored them), those values are used wherever Q_dyn / Z appear:
    in the logits S2 and S3, in Y = P3 Z and in the rowsums; A1 is still
    softmax(Q~ K^T).  That is the gradient of the stored chain with each
    rounding passed through as the identity.
    """
    seeds = np.asarray(seeds, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    dY = np.asarray(dY, dtype=np.float64)
    A1 = attention_weights(seeds, K)  # M x N
    Qd = A1 @ V if Q_dyn is None else np.asarray(Q_dyn, dtype=np.float64)
    A2 = attention_weights(Qd, K)  # M x N
    Zs = A2 @ V if Z is None else np.asarray(Z, dtype=np.float64)
    P3 = attention_weights(K, Qd)  # N x M
    Y = P3 @ Zs

    dZ = P3.T @ dY
    dS3 = _softmax_backward(P3, dY @ Zs.T, np.sum(dY * Y, axis=1))
    dK = dS3 @ Qd
    dQd = dS3.T @ K

    dV = A2.T @ dZ
    dS2 = _softmax_backward(A2, dZ @ V.T, np.sum(dZ * Zs, axis=1))
    dQd = dQd + dS2 @ K
    dK = dK + dS2.T @ Qd

    dV = dV + A1.T @ dQd
    dS1 = _softmax_backward(A1, dQd @ V.T, np.sum(dQd * Qd, axis=1))
    d_seeds = dS1 @ K
    dK = dK + dS1.T @ seeds
    return d_seeds, dK, dV


def flarepp_backward(seeds, K, V, dY, Q_dyn=None, Z=None):
    """Batched backward: seeds [H,M,D], K, V, dY [B,H,N,D] -> (d_seeds [H,M,D],
    dK, dV [B,H,N,D]); the seeds are shared by the batch, so their gradient
    is summed over it.  Q_dyn / Z [B,H,M,D] optionally as stored."""
    B, H, N, D = K.shape
    d_seeds = np.zeros(np.shape(seeds))
    dK = np.zeros((B, H, N, D))
    dV = np.zeros((B, H, N, D))
    for b in range(B):
        for h in range(H):
            g = flarepp_head_backward(seeds[h], K[b, h], V[b, h], dY[b, h],
                                      None if Q_dyn is None else Q_dyn[b, h], None if Z is None else Z[b, h])
            d_seeds[h] += g[0]
            dK[b, h], dV[b, h] = g[1], g[2]
    return d_seeds, dK, dV

