"""The seeded input generators (CPU): determinism, dtype exactness, and the
structure the stress recipes promise the GPU tests."""
import numpy as np

from rank_latent_attention_b200 import inputs


def _bf16_exact(x: np.ndarray) -> bool:
    return bool(np.all((x.astype(np.float32).view(np.uint32) & np.uint32(0xFFFF)) == 0))


def test_workloads_are_deterministic_and_exact():
    for name in ("tiny_f32", "cloud", "long"):
        w = inputs.WORKLOADS[name]
        a, b = inputs.make_inputs(w), inputs.make_inputs(w, threads=1)
        for x, y in zip(a, b):
            assert np.array_equal(x, y), name  # threads do not change the values
        if w.dtype == "bf16":
            assert all(_bf16_exact(x) for x in a), name
    dY = inputs.make_upstream(inputs.WORKLOADS["cloud"])
    assert _bf16_exact(dY) and np.array_equal(dY, inputs.make_upstream(inputs.WORKLOADS["cloud"]))


def test_outlier_rows_scaled():
    w = inputs.WORKLOADS["long"]
    K, V = inputs.make_head(w, 0, 0)
    rows = inputs._outlier_rows(w, 0)
    assert len(rows) == int(np.floor(w.outlier_frac * w.N))
    # the scaled rows stand out by about the outlier gain
    norm = np.linalg.norm(K, axis=1)
    rest = np.setdiff1d(np.arange(w.N), rows)
    assert np.median(norm[rows]) > 0.5 * w.outlier_gain * np.median(norm[rest])


def test_climbing_recipe_keeps_its_promises():
    """inputs.make_climbing drives the encode's skip-max fallback in the GPU
    parity tests; that test means something only if, for every latent, the
    tile maxima climb by more than 6 (log2) per tile on average, so a
    reference set on one tile falls 2^32 behind within six, and the jump tile
    dominates every other token by a wide margin."""
    H, N, jump = 2, 64 * 70 + 37, 50
    for M, D in ((256, 64), (64, 64), (144, 32), (256, 16), (128, 128)):
        Q, K, V = inputs.make_climbing(H, N, M, D, jump_tile=jump)
        assert Q.shape == (H, M, D) and K.shape == V.shape == (1, H, N, D)
        assert _bf16_exact(Q) and _bf16_exact(K) and _bf16_exact(V)
        again = inputs.make_climbing(H, N, M, D, jump_tile=jump)
        assert all(np.array_equal(x, y) for x, y in zip((Q, K, V), again))
        tile = np.arange(N) // 64
        for h in range(H):
            S = Q[h].astype(np.float64) @ K[0, h].astype(np.float64).T * np.log2(np.e)
            tmax = np.stack([S[:, tile == t].max(axis=1) for t in range(jump)], axis=1)  # M x tiles
            climb = (tmax[:, -1] - tmax[:, 0]) / (jump - 1)
            assert np.all(climb > 6.0), (M, D, h, climb.min())
            margin = S[:, tile == jump].max(axis=1) - S[:, tile != jump].max(axis=1)
            assert np.all(margin > 50.0), (M, D, h, margin.min())
