"""Plant plausible mistakes in copies of the oracle and check that the pins catch each.

Every mutant is the oracle's own source with one textual edit, executed as a
fresh module on the CPU.  A mutant that passes every pin would mean the pins
cannot tell that mistake from the definition.
"""
import inspect
import types

import numpy as np
import pytest

import oracle.flare_oracle as base
import oracle_pins

MUTANTS = {
    # scale 1/sqrt(D) instead of the pages' s = 1
    "scale_rsqrt_d": ("return sdpa(Q, K, V, 1.0)", "return sdpa(Q, K, V, 1.0 / np.sqrt(Q.shape[1]))"),
    # encode softmax normalised over the latents instead of the tokens
    "encode_wrong_axis": ("return sdpa(Q, K, V, 1.0)",
                          "return softmax(Q @ K.T, axis=0) @ np.asarray(V, dtype=np.float64)"),
    # sign flip of the logits
    "negated_logits": ("return softmax(scale * (q @ k.T), axis=-1)", "return softmax(-scale * (q @ k.T), axis=-1)"),
    # decode keys taken from Z instead of Q_dyn
    "decode_keys_from_Z": ("Y = flare_decode(K, Q_dyn, Z)", "Y = flare_decode(K, Z, Z)"),
    # decode keys taken from the seeds instead of Q_dyn
    "decode_keys_from_seeds": ("Y = flare_decode(K, Q_dyn, Z)", "Y = flare_decode(K, seeds, Z)"),
    # routing encode driven by the seeds again (no dynamic routing)
    "routing_uses_seeds": ("Z = flare_encode(Q_dyn, K, V)", "Z = flare_encode(seeds, K, V)"),
    # encode values taken from K (dropped V term)
    "encode_values_from_K": ("return sdpa(Q, K, V, 1.0)", "return sdpa(Q, K, K, 1.0)"),
    # decode as the transpose of the encode weights
    "decode_transposed_weights": ("return sdpa(K, Q, Z, 1.0)",
                                  "return attention_weights(Q, K).T @ np.asarray(Z, dtype=np.float64)"),
    # off-by-one in the token index of the values
    "values_shifted": ("return sdpa(Q, K, V, 1.0)", "return sdpa(Q, K, np.roll(V, 1, axis=0), 1.0)"),
    # unnormalised weights (dropped denominator)
    "no_normalisation": ("return E / E.sum(axis=axis, keepdims=True)", "return E"),
    # decode values taken from Q_dyn instead of Z
    "decode_values_qdyn": ("Y = flare_decode(K, Q_dyn, Z)", "Y = flare_decode(K, Q_dyn, Q_dyn)"),
    # the spectral tool using the NxN order of the product
    "eig_wrong_product": ("ev = np.linalg.eigvals(W_enc @ W_dec)", "ev = np.linalg.eigvals(W_enc @ W_enc.T)"),
    # communication matrix built from transposed factors (still NxN)
    "comm_transposed_factors": ("return W_dec @ W_enc", "return W_enc.T @ W_dec.T"),
    # shard log-sum-exp without its max term
    "shard_lse_drops_max": ("return (E @ V) / tot[:, None], top[:, 0] + np.log(tot)",
                            "return (E @ V) / tot[:, None], np.log(tot)"),
    # shards combined as a plain average (statistics ignored)
    "combine_unweighted": ('out[live] = np.einsum("rm,rmd->md", w[:, live], O[:, live]) / tot[live, None]',
                           'out[live] = O[:, live].mean(axis=0)'),
    # shard weights taken linearly in lse instead of exponentially
    "combine_linear_weights": ("w[:, live] = np.exp(lse[:, live] - top[live])",
                               "w[:, live] = 1.0 + lse[:, live] - top[live]"),
    # shard output left unnormalised
    "shard_unnormalised": ("return (E @ V) / tot[:, None], top[:, 0] + np.log(tot)",
                           "return (E @ V), top[:, 0] + np.log(tot)"),
    # decode backward without the softmax's row term
    "bwd_decode_drops_rowsum": ("dS3 = _softmax_backward(P3, dY @ Zs.T, np.sum(dY * Y, axis=1))",
                                "dS3 = _softmax_backward(P3, dY @ Zs.T, 0 * np.sum(dY * Y, axis=1))"),
    # the decode's contribution to dQ_dyn forgotten
    "bwd_no_decode_dqdyn": ("dQd = dS3.T @ K", "dQd = 0 * (dS3.T @ K)"),
    # seed-encode row term taken with Z instead of Q_dyn
    "bwd_seed_rowsum_with_Z": ("np.sum(dQd * Qd, axis=1)", "np.sum(dQd * Zs, axis=1)"),
    # routing-encode value gradient through the decode weights
    "bwd_dv_wrong_weights": ("dV = A2.T @ dZ", "dV = P3 @ dZ"),
    # the seeds' gradient not summed over the batch
    "bwd_seeds_not_summed": ("d_seeds[h] += g[0]", "d_seeds[h] = g[0]"),
    # the seed encode's key gradient taken with Q_dyn
    "bwd_seed_dk_with_qdyn": ("dK = dK + dS1.T @ seeds", "dK = dK + dS1.T @ Qd"),
    # the following three equal the oracle in exact arithmetic and at ordinary
    # logits; they overflow once logits pass float64's exp range
    # softmax without its max shift
    "softmax_no_max_shift": ("E = np.exp(S - S.max(axis=axis, keepdims=True))", "E = np.exp(S)"),
    # shard encode without its max shift (lse then log of the plain sum)
    "shard_no_max_shift": ("E = np.exp(S - top)\n    tot = E.sum(axis=1)\n    return (E @ V) / tot[:, None], top[:, 0] + np.log(tot)",
                           "E = np.exp(S)\n    tot = E.sum(axis=1)\n    return (E @ V) / tot[:, None], np.log(tot)"),
    # shard combine without its max shift
    "combine_no_max_shift": [("w[:, live] = np.exp(lse[:, live] - top[live])", "w[:, live] = np.exp(lse[:, live])"),
                             ("L[live] = top[live] + np.log(tot[live])", "L[live] = np.log(tot[live])")],
}


def _mutant(edits):
    """edits: one (find, replace) pair, or a list of them applied in order."""
    src = inspect.getsource(base)
    for find, repl in ([edits] if isinstance(edits, tuple) else edits):
        assert src.count(find) == 1, f"mutation anchor not unique/absent: {find!r}"
        src = src.replace(find, repl)
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src, "<oracle_mutant>", "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    mod = _mutant(MUTANTS[name])
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            with np.errstate(over="ignore", invalid="ignore", divide="ignore"):  # mutants may overflow
                pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
        except Exception as e:  # a crash on a pin input also exposes the mutant
            caught.append(f"{pin.__name__}:{type(e).__name__}")
    assert caught, f"mutant {name} passed every pin"
