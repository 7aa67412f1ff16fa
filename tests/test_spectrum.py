"""Communication matrix C = W_enc W_dec and its spectrum (flare_communication_matrix)
against the oracle ("FLARE" review page, sections "Матрица коммуникации
низкого ранга" and "Спектральный анализ").

fp32: C within 2e-5 of the fp64 oracle element by element, every row of C
summing to 1 (C is row-stochastic), and the eigenvalues of modulus > 0.05
matching the oracle's within 1e-4, the leading one equal to 1.
bf16: C (bf16 storage; W_dec rounded to bf16 on the way) within
2e-2 RMS(C) + 4 * 2^-9 max|C| of the oracle, rows summing to 1 within 1e-2.
"""
import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from rank_latent_attention_b200 import inputs
from gpu_common import require_cuda, to_dev, to_host

pytestmark = pytest.mark.gpu


def oracle_C(Q, K):
    """[B,H,M,M] fp64: W_enc W_dec per head; Q is [H,M,D] or [B,H,M,D]."""
    B, H = K.shape[:2]
    out = []
    for b in range(B):
        row = []
        for h in range(H):
            q = (Q[h] if Q.ndim == 3 else Q[b, h]).astype(np.float64)
            k = K[b, h].astype(np.float64)
            row.append(oracle.attention_weights(q, k) @ oracle.attention_weights(k, q))
        out.append(np.stack(row))
    return np.stack(out)


def eigenvalues(C):
    """[B,H,M] eigenvalues of each head's C, by decreasing modulus (the caller's
    O(M^3) step: the library returns C only)."""
    ev = np.linalg.eigvals(C)
    return np.take_along_axis(ev, np.argsort(-np.abs(ev), axis=-1), axis=-1)


def match_eigenvalues(got, want, floor):
    """Greedy nearest matching of the eigenvalues of modulus > floor; returns the max distance."""
    want = [w for w in want if abs(w) > floor]
    pool = list(got)
    worst = 0.0
    for w in want:
        j = int(np.argmin([abs(g - w) for g in pool]))
        worst = max(worst, abs(pool[j] - w))
        pool.pop(j)
    return worst


def test_fp32_matrix_and_spectrum():
    torch = require_cuda()
    w = inputs.WORKLOADS["tiny_f32"]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d = to_dev(seeds, "f32"), to_dev(K, "f32")
    C = to_host(flare.flare_communication_matrix(s_d, K_d))
    assert flare.flare_check_status() == (0, 0)
    Co = oracle_C(seeds, K)
    assert np.max(np.abs(C - Co)) < 2e-5
    np.testing.assert_allclose(C.sum(-1), 1.0, atol=2e-5)
    ev = eigenvalues(C)
    for b in range(w.B):
        for h in range(w.H):
            evo = oracle.communication_eigenvalues(seeds[h].astype(np.float64), K[b, h].astype(np.float64))
            assert abs(ev[b, h, 0] - 1.0) < 1e-5
            assert match_eigenvalues(ev[b, h], evo, 0.05) < 1e-4, (b, h)


def test_bf16_routing_queries():
    torch = require_cuda()
    w = inputs.WORKLOADS["cloud"]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, "bf16") for x in (seeds, K, V))
    _, Qd, _ = flare.flarepp_mix_debug(s_d, K_d, V_d)
    C = to_host(flare.flare_communication_matrix(Qd, K_d))
    assert flare.flare_check_status() == (0, 0)
    Co = oracle_C(to_host(Qd), K)  # the GPU's routing queries, as stored (bf16)
    for b in range(w.B):
        for h in range(w.H):
            err = np.max(np.abs(C[b, h] - Co[b, h]))
            lim = 2e-2 * np.sqrt(np.mean(Co[b, h] ** 2)) + 4 * 2.0 ** -9 * np.max(np.abs(Co[b, h]))
            assert err <= lim, (b, h, err, lim)
    np.testing.assert_allclose(C.sum(-1), 1.0, atol=1e-2)


def test_workspace_and_launch_count():
    torch = require_cuda()
    w = inputs.custom(1, 2, 700, 48, 16, dtype="bf16", seed_index=17)
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d = to_dev(seeds, "bf16"), to_dev(K, "bf16")
    nbytes = flare.lib().flare_communication_workspace_size(1, 2, 700, 48, 16, 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    C1 = flare.flare_communication_matrix(s_d, K_d, workspace=ws)
    # ceil(48 / 16) = 3 rounds of identity block, decode, encode + merge, scatter
    assert flare.flare_last_launch_count() == 3 * 5
    C2 = flare.flare_communication_matrix(s_d, K_d)
    assert torch.equal(C1, C2)
    assert flare.flare_check_status() == (0, 0)
