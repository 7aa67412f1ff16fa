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
