"""Communication matrix C = W_enc W_dec and its spectrum (flare_communication_matrix)
against the oracle ("FLARE" review page, sections "Матрица коммуникации
низкого ранга" and "Спектральный анализ").

fp32: C within 2e-5 of the fp64 oracle element by element, every row of C
summing to 1 (C is row-stochastic), and the eigenvalues of modulus > 0.05
matching the oracle's within 1e-4, the leading one equal to 1.
bf16 inputs, one tensor-core pass (M % 16 == 0, D <= 64): both weights are
rounded to fp16 (2^-11 relative; bf16 weights, 2^-9, reached 2.1e-3 on one
eigenvalue of a sharp custom input, fp16 ones 2.5e-4 in a CPU emulation)
and summed in fp32.  With fp32 C (FLARE_BF16_F32OUT): within 4e-3 max|C| of
the oracle per head, rows summing to 1 within 5e-3, the eigenvalues of
modulus > 0.05 within 2e-3.
With bf16 C: within 2e-2 RMS(C) + 4 * 2^-9 max|C|, rows summing to 1 within
1e-2.  The eigen-solve of the M x M matrices is the caller's step (numpy
here).
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
    flare.flare_profile_begin(16)
    C1 = flare.flare_communication_matrix(s_d, K_d, workspace=ws)
    kernels = [k for k, _ in flare.flare_profile_end()]
    # one pass: encode + merge (the per-latent log-sum-exp), the C kernel, the split sum
    assert flare.flare_last_launch_count() == 4
    assert kernels == ["encode_tc", "lse_merge", "comm_tc", "comm_reduce"]
    C2 = flare.flare_communication_matrix(s_d, K_d)
    assert torch.equal(C1, C2)
    assert flare.flare_check_status() == (0, 0)


def _check_f32_C(label, C, Co):
    """fp32 C of the one-pass bf16 path against the oracle, per head."""
    B, H = C.shape[:2]
    for b in range(B):
        for h in range(H):
            err = np.max(np.abs(C[b, h] - Co[b, h]))
            lim = 4e-3 * np.max(np.abs(Co[b, h]))
            assert err <= lim, (label, b, h, err, lim)
            assert np.max(np.abs(C[b, h].sum(-1) - 1.0)) <= 5e-3, (label, b, h)
            evo = np.linalg.eigvals(Co[b, h])
            assert match_eigenvalues(eigenvalues(C[b, h][None, None])[0, 0], evo, 0.05) <= 2e-3, (label, b, h)


@pytest.mark.parametrize("name", ["cloud", "mesh2d", "long"])
def test_fp32_matrix_from_bf16_routing_queries(name):
    """fp32 C from bf16 inputs in one pass, with the GPU's own routing queries."""
    torch = require_cuda()
    w = inputs.WORKLOADS[name]
    seeds, K, V = inputs.make_inputs(w)
    nb = min(w.B, 2)  # two batch elements keep the oracle quick
    s_d, K_d, V_d = (to_dev(x, "bf16") for x in (seeds, K[:nb], V[:nb]))
    _, Qd, _ = flare.flarepp_mix_debug(s_d, K_d, V_d)
    C = flare.flare_communication_matrix(Qd, K_d, out_dtype=torch.float32)
    assert C.dtype == torch.float32 and flare.flare_check_status() == (0, 0)
    _check_f32_C(name, to_host(C), oracle_C(to_host(Qd), K[:nb]))


@pytest.mark.parametrize("B,H,N,M,D", [(1, 1, 1, 16, 16), (1, 2, 127, 48, 32), (2, 1, 1000, 144, 64),
                                       (1, 2, 5000, 256, 64), (1, 1, 40000, 256, 32), (1, 3, 333, 128, 16)])
def test_fp32_matrix_shapes(B, H, N, M, D):
    """Ragged and one-token heads, both latent-count forms (M <= 128, M > 128), several token splits."""
    torch = require_cuda()
    w = inputs.custom(B, H, N, M, D, dtype="bf16", scale=0.6)
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d = to_dev(seeds, "bf16"), to_dev(K, "bf16")
    C = flare.flare_communication_matrix(s_d, K_d, out_dtype=torch.float32)
    assert flare.flare_check_status() == (0, 0)
    _check_f32_C(f"{(B, H, N, M, D)}", to_host(C), oracle_C(seeds, K))


def test_split_counts_agree():
    """The sum over token splits makes C independent of the split count: each
    count matches the oracle, and they agree to the fp16 rounding of the
    weights (the override also moves the encode's split count, hence the last
    bits of the per-latent log-sum-exp, and a weight can round the other way)."""
    torch = require_cuda()
    w = inputs.custom(1, 2, 3000, 256, 32, dtype="bf16", scale=0.6)
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d = to_dev(seeds, "bf16"), to_dev(K, "bf16")
    Co = oracle_C(seeds, K)
    outs = []
    for splits in (1, 3, 1000):
        old = flare.flare_set_split_override(splits)
        try:
            outs.append(to_host(flare.flare_communication_matrix(s_d, K_d, out_dtype=torch.float32)))
        finally:
            flare.flare_set_split_override(old)
        _check_f32_C(f"splits={splits}", outs[-1], Co)
    assert flare.flare_check_status() == (0, 0)
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 2.0 ** -11 * np.max(np.abs(outs[0]))
