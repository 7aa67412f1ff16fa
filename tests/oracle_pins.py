"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``pin_*`` function takes an oracle module ``o`` and raises AssertionError
when ``o`` disagrees with the reference it pins against.  ``tests/test_oracle.py``
runs every pin on the real oracle; ``tests/test_oracle_mutations.py`` plants
plausible mistakes in copies of the oracle's source and checks that each
mistake fails at least one pin.

What pins what:

* worked examples (``tests/golden/worked_examples.json``): hand-derived exact
  fractions for the chained FLARE++ head (composition, operand roles, scale,
  softmax axes).
* torch float64 SDPA: each of ``flare_encode`` / ``flare_decode`` is one SDPA
  call with scale 1 ("FLARE" review page, "Основной механизм FLARE").
* pure-Python brute force: scalar loops with ``math.exp`` following the
  definitions, independent of NumPy.
* dense construction: explicit W_encode (MxN) and W_decode (NxM) from the
  "Матрица коммуникации низкого ранга" section; the FLARE output is W V.
* rank and spectrum: W has numerical rank <= M; its nonzero eigenvalues are
  those of W_encode W_decode ("Спектральный анализ").
* invariants of the definition: row sums, K = 0, M = 1, N = 1, constant V,
  token permutation, key shift, convex hull.
* token shards ("FLARE++" page, "Contributions Clés", context parallelism):
  the shard results combined equal the pure-Python encode over all tokens;
  each shard's log-sum-exp equals a scalar ``math.log(fsum(exp))`` and
  scipy's ``logsumexp``; one-token and empty shards take their closed forms.
* logits past float64's exp range (up to ~1.3e3, the regime the softmaxes'
  max shift exists for): the encode against the pure-Python brute force and
  against the encode over the dominant tokens alone; the shards' lse against
  scipy's logsumexp; the combined shards; the chained head finite and inside
  the values' hull.
* backward: torch float64 autograd through three SDPA calls; central finite
  differences of the oracle's own forward along random directions; closed
  forms (N = 1: dV = dY, dK = 0, d_seeds = 0; K = 0: dV = mean of dY,
  d_seeds = 0); the seeds' gradient summed over the batch; the
  stored-intermediates form equal to the exact one when given the exact
  intermediates.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _rng(seed):
    return np.random.default_rng(seed)


def _case(seed, N, M, D, std=0.7):
    g = _rng(seed)
    return (g.standard_normal((M, D)) * std, g.standard_normal((N, D)) * std,
            g.standard_normal((N, D)) * std)


# ---------------------------------------------------------------- worked examples
def _parse_key(s: str) -> float:
    s = s.strip()
    if s.startswith("ln(") and s.endswith(")"):
        return math.log(float(Fraction(s[3:-1])))
    return float(Fraction(s))


def _frac(s: str) -> float:
    return float(Fraction(s))


def pin_worked_examples(o):
    with open(GOLDEN) as f:
        data = json.load(f)
    for ex in data["examples"]:
        seeds = np.array([[_parse_key(x) for x in r] for r in ex["seeds"]])
        K = np.array([[_parse_key(x) for x in r] for r in ex["K"]])
        V = np.array([[_parse_key(x) for x in r] for r in ex["V"]])
        Qd, Z, Y = o.flarepp_head(seeds, K, V)
        for name, got in (("Q_dyn", Qd), ("Z", Z), ("Y", Y)):
            want = np.array([[_frac(x) for x in r] for r in ex[name]])
            assert got.shape == want.shape, (ex["name"], name, got.shape, want.shape)
            assert np.allclose(got, want, rtol=1e-13, atol=1e-13), (ex["name"], name, got, want)


# ---------------------------------------------------------------- torch SDPA
def pin_torch_sdpa(o):
    import torch
    import torch.nn.functional as F

    for seed, (N, M, D) in enumerate([(37, 5, 3), (200, 16, 8), (129, 1, 4), (1, 3, 2), (64, 64, 16)]):
        Q, K, V = _case(100 + seed, N, M, D)
        tq, tk, tv = (torch.from_numpy(x) for x in (Q, K, V))
        want_enc = F.scaled_dot_product_attention(tq[None], tk[None], tv[None], scale=1.0)[0].numpy()
        got_enc = o.flare_encode(Q, K, V)
        assert np.allclose(got_enc, want_enc, rtol=1e-12, atol=1e-13), ("encode", N, M, D)
        Zl = _rng(200 + seed).standard_normal((M, D))
        want_dec = F.scaled_dot_product_attention(tk[None], tq[None], torch.from_numpy(Zl)[None],
                                                  scale=1.0)[0].numpy()
        got_dec = o.flare_decode(K, Q, Zl)
        assert np.allclose(got_dec, want_dec, rtol=1e-12, atol=1e-13), ("decode", N, M, D)


# ---------------------------------------------------------------- brute force
def _bf_encode(Q, K, V):
    M, N, D = len(Q), len(K), len(V[0])
    out = []
    for m in range(M):
        logits = [sum(Q[m][d] * K[n][d] for d in range(len(K[0]))) for n in range(N)]
        top = max(logits)
        w = [math.exp(x - top) for x in logits]
        tot = math.fsum(w)
        out.append([math.fsum(w[n] * V[n][d] for n in range(N)) / tot for d in range(D)])
    return out


def _bf_decode(K, Q, Z):
    N, M, D = len(K), len(Q), len(Z[0])
    out = []
    for n in range(N):
        logits = [sum(K[n][d] * Q[m][d] for d in range(len(K[0]))) for m in range(M)]
        top = max(logits)
        w = [math.exp(x - top) for x in logits]
        tot = math.fsum(w)
        out.append([math.fsum(w[m] * Z[m][d] for m in range(M)) / tot for d in range(D)])
    return out


def brute_force_head(seeds, K, V):
    seeds, K, V = seeds.tolist(), K.tolist(), V.tolist()
    Qd = _bf_encode(seeds, K, V)
    Z = _bf_encode(Qd, K, V)
    Y = _bf_decode(K, Qd, Z)
    return np.array(Qd), np.array(Z), np.array(Y)


def pin_brute_force(o):
    for seed, (N, M, D) in enumerate([(1, 1, 1), (2, 1, 2), (5, 3, 2), (8, 4, 3), (7, 2, 1), (6, 4, 4)]):
        S, K, V = _case(300 + seed, N, M, D, std=1.1)
        want = brute_force_head(S, K, V)
        got = o.flarepp_head(S, K, V)
        for name, g, w in zip(("Q_dyn", "Z", "Y"), got, want):
            assert np.allclose(g, w, rtol=1e-12, atol=1e-13), (name, N, M, D)


# ---------------------------------------------------------------- dense NxN operator
def _bf_weights(A, B):
    """softmax over the rows of B of A B^T, by scalar loops."""
    out = []
    for a in A:
        logits = [sum(x * y for x, y in zip(a, b)) for b in B]
        top = max(logits)
        w = [math.exp(x - top) for x in logits]
        tot = math.fsum(w)
        out.append([x / tot for x in w])
    return np.array(out)


def pin_dense_operator(o):
    for seed, (N, M, D) in enumerate([(12, 3, 2), (40, 5, 4), (9, 9, 3)]):
        Q, K, V = _case(400 + seed, N, M, D)
        W_enc = _bf_weights(Q.tolist(), K.tolist())  # M x N
        W_dec = _bf_weights(K.tolist(), Q.tolist())  # N x M
        W = W_dec @ W_enc
        assert np.allclose(o.communication_matrix(Q, K), W, rtol=1e-12, atol=1e-14)
        Z = o.flare_encode(Q, K, V)
        assert np.allclose(Z, W_enc @ V, rtol=1e-12, atol=1e-13)
        Y = o.flare_decode(K, Q, Z)
        assert np.allclose(Y, W @ V, rtol=1e-12, atol=1e-13)
        assert np.allclose(o.attention_weights(Q, K), W_enc, rtol=1e-12, atol=1e-14)


def pin_rank_and_spectrum(o):
    for seed, (N, M, D) in enumerate([(64, 4, 8), (48, 7, 3)]):
        Q, K, _ = _case(500 + seed, N, M, D, std=1.0)
        W = o.communication_matrix(Q, K)
        sv = np.linalg.svd(W, compute_uv=False)
        assert sv[M] / sv[0] < 1e-12, ("rank", sv[: M + 2])
        assert np.allclose(W.sum(axis=1), 1.0, atol=1e-13)  # row-stochastic
        ev_small = o.communication_eigenvalues(Q, K)
        ev_big = np.linalg.eigvals(W)
        ev_big = ev_big[np.argsort(-np.abs(ev_big))][:M]
        assert np.allclose(np.sort_complex(ev_small), np.sort_complex(ev_big), atol=1e-10), (ev_small, ev_big)
        assert abs(ev_small[0] - 1.0) < 1e-10  # W 1 = 1, and W_enc W_dec is row-stochastic too


# ---------------------------------------------------------------- invariants
def pin_invariants(o):
    N, M, D = 50, 6, 4
    S, K, V = _case(600, N, M, D, std=0.9)

    # every attention row sums to one, for all three steps
    Qd, Z, Y = o.flarepp_head(S, K, V)
    for A in (o.attention_weights(S, K), o.attention_weights(Qd, K), o.attention_weights(K, Qd)):
        assert np.allclose(A.sum(axis=1), 1.0, atol=1e-13)

    # K = 0: every encode weight is 1/N, so Q_dyn = Z = mean(V), and Y rows = mean(V)
    mean = V.mean(axis=0)
    Qd0, Z0, Y0 = o.flarepp_head(S, np.zeros_like(K), V)
    assert np.allclose(Qd0, mean[None], atol=1e-13)
    assert np.allclose(Z0, mean[None], atol=1e-13)
    assert np.allclose(Y0, mean[None], atol=1e-13)

    # M = 1: the decode softmax over one latent is 1, so every Y row equals Z
    Qd1, Z1, Y1 = o.flarepp_head(S[:1], K, V)
    assert np.allclose(Y1, Z1[0][None], atol=1e-13)

    # N = 1: every softmax over tokens picks the single token
    Qdn, Zn, Yn = o.flarepp_head(S, K[:1], V[:1])
    assert np.allclose(Qdn, V[:1], atol=1e-13) and np.allclose(Zn, V[:1], atol=1e-13)
    assert np.allclose(Yn, V[:1], atol=1e-13)

    # constant V: every convex combination returns that constant
    c = _rng(601).standard_normal(D)
    _, _, Yc = o.flarepp_head(S, K, np.tile(c, (N, 1)))
    assert np.allclose(Yc, c[None], atol=1e-13)

    # token permutation: Q_dyn and Z unchanged, Y permuted the same way
    p = _rng(602).permutation(N)
    Qdp, Zp, Yp = o.flarepp_head(S, K[p], V[p])
    assert np.allclose(Qdp, Qd, atol=1e-13) and np.allclose(Zp, Z, atol=1e-13)
    assert np.allclose(Yp, Y[p], atol=1e-13)

    # key shift K -> K + 1 u^T: each encode row's logits move by a constant
    u = _rng(603).standard_normal(D)
    Qds, Zs, Ys = o.flarepp_head(S, K + u[None], V)
    assert np.allclose(Qds, Qd, atol=1e-12) and np.allclose(Zs, Z, atol=1e-12)
    assert not np.allclose(Ys, Y, atol=1e-6)  # the decode is not shift invariant

    # decode query shift Q -> Q + 1 c^T leaves the decode weights unchanged
    cq = _rng(604).standard_normal(D)
    assert np.allclose(o.flare_decode(K, Qd + cq[None], Z), o.flare_decode(K, Qd, Z), atol=1e-12)

    # convex hull: every output lies within [min_n V, max_n V] per channel
    lo, hi = V.min(axis=0), V.max(axis=0)
    for X in (Qd, Z, Y):
        assert np.all(X >= lo - 1e-13) and np.all(X <= hi + 1e-13)


def pin_mix_layout(o):
    """flarepp_mix applies one head's chain per (b, h) with seeds shared over the batch."""
    B, H, N, M, D = 2, 3, 11, 4, 2
    g = _rng(700)
    seeds = g.standard_normal((H, M, D))
    K = g.standard_normal((B, H, N, D))
    V = g.standard_normal((B, H, N, D))
    Qd, Z, Y = o.flarepp_mix(seeds, K, V)
    for b in range(B):
        for h in range(H):
            want = brute_force_head(seeds[h], K[b, h], V[b, h])
            for got, w in zip((Qd[b, h], Z[b, h], Y[b, h]), want):
                assert np.allclose(got, w, rtol=1e-12, atol=1e-13), (b, h)
    rows = [0, 5, 10]
    Yr = o.flarepp_decode_rows(K[1, 2], Qd[1, 2], Z[1, 2], rows)
    assert np.allclose(Yr, Y[1, 2][rows], atol=1e-14)


# ---------------------------------------------------------------- token shards
def _bf_lse(Q, K):
    out = []
    for q in Q:
        logits = [sum(q[d] * k[d] for d in range(len(q))) for k in K]
        top = max(logits)
        out.append(top + math.log(math.fsum(math.exp(x - top) for x in logits)))
    return out


def pin_shard_combine(o):
    from scipy.special import logsumexp

    for seed, (N, M, D, cuts) in enumerate([(7, 3, 2, [0, 3, 3, 7]), (12, 4, 3, [0, 1, 5, 11, 12]),
                                            (5, 2, 2, [0, 5]), (9, 1, 1, [0, 0, 4, 9, 9])]):
        Q, K, V = _case(800 + seed, N, M, D, std=1.3)
        parts = [o.encode_shard(Q, K[a:b], V[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
        for (Op, lp), a, b in zip(parts, cuts[:-1], cuts[1:]):
            if b == a:  # empty shard: no tokens, no weight
                assert np.all(Op == 0) and np.all(np.isneginf(lp)), ("empty", seed)
                continue
            assert np.allclose(lp, _bf_lse(Q.tolist(), K[a:b].tolist()), rtol=1e-13, atol=1e-13), ("lse", seed)
            assert np.allclose(lp, logsumexp(Q @ K[a:b].T, axis=1), rtol=1e-13, atol=1e-13), ("lse", seed)
            assert np.allclose(Op, _bf_encode(Q.tolist(), K[a:b].tolist(), V[a:b].tolist()), rtol=1e-12,
                               atol=1e-13), ("O", seed)
            if b - a == 1:  # one token: O is its value row, lse its logit
                assert np.allclose(Op, np.broadcast_to(V[a], Op.shape), atol=1e-15)
                assert np.allclose(lp, Q @ K[a], atol=1e-14)
        out, L = o.combine_shards([p[0] for p in parts], [p[1] for p in parts])
        assert np.allclose(out, _bf_encode(Q.tolist(), K.tolist(), V.tolist()), rtol=1e-12, atol=1e-13), seed
        assert np.allclose(L, logsumexp(Q @ K.T, axis=1), rtol=1e-13, atol=1e-13), seed
        rev, Lr = o.combine_shards([p[0] for p in parts[::-1]], [p[1] for p in parts[::-1]])
        assert np.allclose(rev, out, atol=1e-14) and np.allclose(Lr, L, atol=1e-14), seed
    # a latent with every shard empty
    out, L = o.combine_shards([np.zeros((2, 3))] * 2, [np.full(2, -np.inf)] * 2)
    assert np.all(out == 0) and np.all(np.isneginf(L))


# ---------------------------------------------------------------- extreme logits
def _extreme_case(seed, N=48, M=3, D=4):
    """Logits that climb by ~25 per token past float64's exp range (up to
    ~1.3e3), a block of four tokens (40-43) 200 above the climb, and the
    tokens after it 400 below: only a max-shifted softmax stays finite."""
    g = _rng(seed)
    e = g.standard_normal(D)
    e /= np.linalg.norm(e)
    Q = e[None, :] + 0.02 * g.standard_normal((M, D))
    a = 25.0 * np.arange(N, dtype=np.float64)
    a[40:44] += 200.0
    a[44:] -= 400.0
    K = a[:, None] * e[None, :] + 0.02 * g.standard_normal((N, D))
    V = g.standard_normal((N, D))
    return Q, K, V


def pin_extreme_logits(o):
    from scipy.special import logsumexp

    Q, K, V = _extreme_case(1100)
    S = Q @ K.T
    assert S.max() > 1000.0  # exp of it overflows float64
    Z = o.flare_encode(Q, K, V)
    assert np.all(np.isfinite(Z))
    assert np.allclose(Z, _bf_encode(Q.tolist(), K.tolist(), V.tolist()), rtol=1e-12, atol=1e-13)
    # every token outside 40-43 sits at least ~180 below them (weight below
    # e^-180 of theirs): the encode over those four tokens alone agrees
    assert np.allclose(Z, o.flare_encode(Q, K[40:44], V[40:44]), rtol=1e-13, atol=1e-14)
    assert np.allclose(o.attention_weights(Q, K).sum(axis=1), 1.0, atol=1e-13)
    cuts = [0, 16, 40, 48]
    parts = [o.encode_shard(Q, K[a:b], V[a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
    for (Op, lp), a, b in zip(parts, cuts[:-1], cuts[1:]):
        assert np.all(np.isfinite(Op)) and np.all(np.isfinite(lp)), ("shard", a, b)
        assert np.allclose(lp, logsumexp(S[:, a:b], axis=1), rtol=1e-14, atol=1e-11), ("lse", a, b)
        assert np.allclose(lp, _bf_lse(Q.tolist(), K[a:b].tolist()), rtol=1e-14, atol=1e-11), ("lse", a, b)
    out, L = o.combine_shards([p[0] for p in parts], [p[1] for p in parts])
    assert np.allclose(out, Z, rtol=1e-12, atol=1e-13)
    assert np.allclose(L, logsumexp(S, axis=1), rtol=1e-14, atol=1e-11)
    # the chained head: routing and decode logits grow larger still
    Qd, Zh, Y = o.flarepp_head(Q, K, V)
    lo, hi = V.min(axis=0), V.max(axis=0)
    for X in (Qd, Zh, Y):
        assert np.all(np.isfinite(X)) and np.all(X >= lo - 1e-12) and np.all(X <= hi + 1e-12)


# ---------------------------------------------------------------- backward
def _torch_chain_grads(seeds, K, V, dY):
    import torch

    F = torch.nn.functional.scaled_dot_product_attention
    t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (seeds, K, V)]
    Qd = F(t[0][None], t[1][None], t[2][None], scale=1.0)[0]
    Z = F(Qd[None], t[1][None], t[2][None], scale=1.0)[0]
    Y = F(t[1][None], Qd[None], Z[None], scale=1.0)[0]
    (Y * torch.tensor(dY, dtype=torch.float64)).sum().backward()
    return [x.grad.numpy() for x in t]


def pin_backward(o):
    for seed, (N, M, D) in enumerate([(7, 3, 4), (12, 5, 2), (4, 4, 3), (9, 1, 2), (3, 6, 5)]):
        S, K, V = _case(900 + seed, N, M, D, std=0.9)
        dY = _rng(950 + seed).standard_normal((N, D))
        got = o.flarepp_head_backward(S, K, V, dY)
        for name, g, w in zip(("d_seeds", "dK", "dV"), got, _torch_chain_grads(S, K, V, dY)):
            assert np.allclose(g, w, rtol=1e-10, atol=1e-12), ("autograd", name, N, M, D)
        # directional finite differences of L = sum(dY * Y) through the forward
        g = _rng(980 + seed)
        U = [g.standard_normal(x.shape) for x in (S, K, V)]
        eps = 1e-5

        def L(t):
            return float(np.sum(dY * o.flarepp_head(S + t * U[0], K + t * U[1], V + t * U[2])[2]))

        fd = (L(eps) - L(-eps)) / (2 * eps)
        an = sum(float(np.sum(gi * ui)) for gi, ui in zip(got, U))
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), ("finite differences", fd, an)
        # the stored-intermediates form, given the exact intermediates
        Qd, Z, _ = o.flarepp_head(S, K, V)
        again = o.flarepp_head_backward(S, K, V, dY, Q_dyn=Qd, Z=Z)
        for a, b in zip(got, again):
            assert np.allclose(a, b, rtol=1e-13, atol=1e-14)
    # N = 1: Y = V whatever the seeds and keys
    S, K, V = _case(990, 1, 3, 2)
    dY = _rng(991).standard_normal((1, 2))
    ds, dk, dv = o.flarepp_head_backward(S, K, V, dY)
    assert np.allclose(ds, 0, atol=1e-15) and np.allclose(dk, 0, atol=1e-15) and np.allclose(dv, dY, atol=1e-15)
    # K = 0: every softmax is uniform, Y = mean(V), the seeds have no effect
    S, _, V = _case(992, 6, 3, 2)
    dY = _rng(993).standard_normal((6, 2))
    ds, dk, dv = o.flarepp_head_backward(S, np.zeros((6, 2)), V, dY)
    assert np.allclose(dv, np.broadcast_to(dY.mean(axis=0), dv.shape), atol=1e-14)
    assert np.allclose(ds, 0, atol=1e-15)
    # batched form: seeds shared by the batch, their gradient summed over it
    B, H, N, M, D = 2, 2, 5, 3, 2
    g = _rng(994)
    seeds = g.standard_normal((H, M, D))
    K, V, dY = (g.standard_normal((B, H, N, D)) for _ in range(3))
    ds, dk, dv = o.flarepp_backward(seeds, K, V, dY)
    for h in range(H):
        want = [_torch_chain_grads(seeds[h], K[b, h], V[b, h], dY[b, h]) for b in range(B)]
        assert np.allclose(ds[h], want[0][0] + want[1][0], rtol=1e-10, atol=1e-12)
        for b in range(B):
            assert np.allclose(dk[b, h], want[b][1], rtol=1e-10, atol=1e-12)
            assert np.allclose(dv[b, h], want[b][2], rtol=1e-10, atol=1e-12)


ALL_PINS = [
    pin_worked_examples,
    pin_torch_sdpa,
    pin_brute_force,
    pin_dense_operator,
    pin_rank_and_spectrum,
    pin_invariants,
    pin_mix_layout,
    pin_shard_combine,
    pin_extreme_logits,
    pin_backward,
]
