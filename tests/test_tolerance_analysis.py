"""Why the stated bf16 bar cannot hold for every workload with bf16 storage (CPU only).

The stated bar for bf16 inputs is max|Y - Y_oracle| <= 2e-2 * RMS(Y_oracle).
With 1% of tokens scaled x8 in K and V ("long" workload), a few decode rows
are sharp averages of large Z rows while most rows average to small values,
so max|Y| is tens of times RMS(Y).  Rounding the oracle's own fp64 Y to bf16
(half an ulp is 2^-9 relative) then already breaks the bar: no kernel that
stores Y as bf16 can meet it there, which is why the library also offers
bf16 inputs with fp32 arithmetic and fp32 Y.  On the Gaussian workloads the
same rounding stays well inside the bar.
"""
import numpy as np
import torch

import oracle
from rank_latent_attention_b200 import inputs


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _oracle_Y(w, heads):
    seeds, K, V = inputs.make_inputs(w)
    return np.stack([oracle.flarepp_head(seeds[h].astype(np.float64), K[b, h].astype(np.float64),
                                         V[b, h].astype(np.float64))[2] for b, h in heads])


def test_bf16_rounding_of_exact_output_breaks_bar_on_outlier_workload():
    w = inputs.WORKLOADS["long"]
    Y = _oracle_Y(w, [(b, h) for b in range(6) for h in range(w.H)])
    rms = np.sqrt(np.mean(Y ** 2))
    err = np.max(np.abs(_bf16(Y) - Y))
    assert np.max(np.abs(Y)) > 10 * rms
    assert err > 2e-2 * rms, (err, rms)


def test_bf16_rounding_of_exact_output_fits_bar_on_gaussian_workloads():
    for w, heads in ((inputs.WORKLOADS["cloud"], [(b, h) for b in range(2) for h in range(8)]),
                     (inputs.custom(1, 2, 1 << 15, 256, 64), [(0, 0), (0, 1)])):
        Y = _oracle_Y(w, heads)
        rms = np.sqrt(np.mean(Y ** 2))
        assert np.max(np.abs(_bf16(Y) - Y)) < 0.5 * 2e-2 * rms


def _chain_with_bf16_storage(seeds, K, V):
    """The three steps computed exactly, with Q_dyn, Z and Y stored as bf16
    between them: what three chained bf16 SDPA calls return."""
    q = _bf16(oracle.flare_encode(seeds, K, V))
    z = _bf16(oracle.flare_encode(q, K, V))
    return _bf16(oracle.flare_decode(K, q, z))


def test_bf16_storage_of_the_chain_breaks_bar_on_mesh_workload():
    """On the smooth-field mesh workload the bf16 storage of the intermediates
    alone (exact arithmetic otherwise) already exceeds 2e-2 x RMS(Y): rounding
    Q_dyn moves the decode logits of these large-norm keys, and no kernel that
    keeps Q_dyn and Z in bf16 can meet the stated bar there.  The split-
    precision mode (hi/lo bf16 pairs, fp32 output) is what meets it."""
    w = inputs.WORKLOADS["mesh2d"]
    seeds, K, V = (x.astype(np.float64) for x in inputs.make_inputs(w))
    heads = [(b, h) for b in range(w.B) for h in range(w.H)]
    Y = np.stack([oracle.flarepp_head(seeds[h], K[b, h], V[b, h])[2] for b, h in heads])
    G = np.stack([_chain_with_bf16_storage(seeds[h], K[b, h], V[b, h]) for b, h in heads])
    rms = np.sqrt(np.mean(Y ** 2))
    assert np.max(np.abs(G - Y)) > 1.1 * 2e-2 * rms
    # the rounding of Y itself is not the cause: the exact Y rounded fits
    assert np.max(np.abs(_bf16(Y) - Y)) < 0.9 * 2e-2 * rms


def test_bf16_storage_of_the_chain_fits_bar_on_gaussian_cloud():
    w = inputs.WORKLOADS["cloud"]
    seeds, K, V = (x.astype(np.float64) for x in inputs.make_inputs(w))
    heads = [(b, h) for b in range(4) for h in range(w.H)]
    Y = np.stack([oracle.flarepp_head(seeds[h], K[b, h], V[b, h])[2] for b, h in heads])
    G = np.stack([_chain_with_bf16_storage(seeds[h], K[b, h], V[b, h]) for b, h in heads])
    assert np.max(np.abs(G - Y)) < 0.6 * 2e-2 * np.sqrt(np.mean(Y ** 2))
