"""GPU parity of flarepp_mix_backward against the fp64 oracle's backward.

Two references per case:
* stored: oracle.flarepp_backward given the Q_dyn and Z the GPU forward
  stored (flarepp_mix_debug) -- the gradient of the computed chain with each
  rounding taken as the identity, which is what the library computes.
* exact: the oracle's exact gradient.  On fp32 inputs it is the same as the
  stored one; on bf16 the stored Q_dyn and Z sit one bf16 rounding away.
Bars: tests/gpu_common.py, assert_backward_bar (CUDA-core kernels 1e-4 x
RMS; tensor-core kernels 2e-2 x RMS + 16 x 2^-9 x the head's max|gradient|),
the same for both references.
"""
import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from gpu_common import assert_backward_bar, encode_kernels, require_cuda, rms, to_dev, to_host
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu

NAMES = ("d_seeds", "dK", "dV")
CASES = [
    ("tiny_f32", None),
    ("cloud", None),
    ("custom", (2, 3, 333, 48, 32, "f32")),     # ragged tokens, M not a multiple of 32
    ("custom", (1, 2, 517, 256, 128, "bf16")),  # largest M and D
    ("custom", (3, 2, 1, 16, 16, "bf16")),      # N = 1: dV = dY, the rest 0
    ("custom", (1, 1, 100, 1, 16, "f32")),      # M = 1
    ("custom", (2, 2, 257, 64, 64, "bf16")),
    ("custom", (2, 2, 300, 48, 32, "bf16")),    # tensor cores, M not a multiple of 32
    ("custom", (1, 3, 1000, 16, 64, "bf16")),   # one 16-latent chunk
    ("custom", (1, 2, 700, 256, 64, "bf16")),   # both latent halves, the benchmark's M and D
    ("long2", None),                            # heavy-tailed: 1% of tokens x8 (two batch elements)
]


def _workload(name, spec):
    if name == "long2":
        import dataclasses
        return dataclasses.replace(inputs.WORKLOADS["long"], B=2)
    if name != "custom":
        return inputs.WORKLOADS[name]
    B, H, N, M, D, dt = spec
    return inputs.custom(B, H, N, M, D, dtype=dt, seed_index=70 + N % 17)


def _run(w):
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    dev = [to_dev(x, w.dtype) for x in (seeds, K, V, dY)]
    grads = flare.flarepp_mix_backward(*dev)
    launches = flare.flare_last_launch_count()
    _, Qd, Z = flare.flarepp_mix_debug(*dev[:3])
    assert flare.flare_check_status() == (0, 0)
    return (seeds, K, V, dY), [to_host(g) for g in grads], to_host(Qd), to_host(Z), launches


def _excess(got, want, rel):
    """max over elements of (|got - want| - rel |want|) / RMS(want), per gradient."""
    return [float(np.max(np.abs(g - r) - rel * np.abs(r))) / max(rms(r), 1e-30) for g, r in zip(got, want)]


@pytest.mark.parametrize("name,spec", CASES, ids=lambda x: str(x))
def test_backward_matches_oracle(name, spec):
    require_cuda()
    w = _workload(name, spec)
    (seeds, K, V, dY), got, Qd, Z, launches = _run(w)
    # the two recomputed encodes (each with its merge unless it runs one CTA
    # per head) + eight backward kernels
    assert launches == 2 * len(encode_kernels(w.B, w.H, w.N, w.dtype == "bf16")) + 8
    args = [x.astype(np.float64) for x in (seeds, K, V, dY)]
    stored = oracle.flarepp_backward(*args, Q_dyn=Qd, Z=Z)
    exact = stored if w.dtype == "f32" else oracle.flarepp_backward(*args)
    rel = 0.0 if w.dtype == "f32" else 2.0 ** -8  # the bf16 store of each gradient
    e_stored, e_exact = _excess(got, stored, rel), _excess(got, exact, rel)
    print(f"{w.name}: stored {e_stored} exact {e_exact}")
    for g in got:
        assert np.all(np.isfinite(g))
    if w.N == 1:  # Y = V: dV = dY (up to its bf16 store), nothing else moves Y
        assert np.allclose(got[2], dY, rtol=2.0 ** -8, atol=1e-6)
        assert np.max(np.abs(got[0])) <= 1e-4 and np.max(np.abs(got[1])) <= 1e-4
        return
    tensor_cores = w.dtype == "bf16" and w.D <= 64
    for n, g, r in zip(NAMES, got, stored):
        assert_backward_bar(f"{w.name}.{n}.stored", g, r, w.dtype, tensor_cores)
    if w.dtype == "bf16":
        for n, g, r in zip(NAMES, got, exact):
            assert_backward_bar(f"{w.name}.{n}.exact", g, r, w.dtype, True)


@pytest.mark.parametrize("spec", [(1, 2, 64 * 13 + 5, 256, 64), (1, 2, 64 * 9 + 33, 144, 32),
                                  (2, 1, 64 * 7 + 1, 48, 16)], ids=str)
def test_backward_many_tiles_per_cta(spec):
    """One and three token splits per head: every backward kernel runs several
    token tiles per CTA (14, 10 and 8 of the latent kernel's 64 tokens at one
    split), so its stage rings wrap -- four stages in the encode part, two in
    the decode part -- and the ragged last tile comes after full ones.  The
    default split rule gives these sizes one tile per CTA."""
    require_cuda()
    B, H, N, M, D = spec
    w = inputs.custom(B, H, N, M, D, dtype="bf16", seed_index=90 + N % 13)
    exact = None
    for splits in (1, 3):
        old = flare.flare_set_split_override(splits)
        try:
            (seeds, K, V, dY), got, Qd, Z, _ = _run(w)
        finally:
            flare.flare_set_split_override(old)
        args = [x.astype(np.float64) for x in (seeds, K, V, dY)]
        stored = oracle.flarepp_backward(*args, Q_dyn=Qd, Z=Z)
        if exact is None:
            exact = oracle.flarepp_backward(*args)
        print(f"{spec} splits={splits}: stored {_excess(got, stored, 2.0 ** -8)} exact {_excess(got, exact, 2.0 ** -8)}")
        for n, g, r in zip(NAMES, got, stored):
            assert np.all(np.isfinite(g))
            assert_backward_bar(f"{spec}/{splits}.{n}.stored", g, r, "bf16", True)
        for n, g, r in zip(NAMES, got, exact):
            assert_backward_bar(f"{spec}/{splits}.{n}.exact", g, r, "bf16", True)


def test_workspace_and_stream():
    import torch

    require_cuda()
    w = inputs.custom(1, 2, 300, 32, 32, dtype="bf16", seed_index=77)
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    dev = [to_dev(x, "bf16") for x in (seeds, K, V, dY)]
    nbytes = flare.flarepp_mix_backward_workspace_size(1, 2, 300, 32, 32, torch.bfloat16)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g1 = flare.flarepp_mix_backward(*dev, workspace=ws, stream=s)
    s.synchronize()
    g2 = flare.flarepp_mix_backward(*dev)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)  # same kernels, same order: the same bits
    small = torch.empty(nbytes - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(flare.FlareError):
        flare.flarepp_mix_backward(*dev, workspace=small)


@pytest.mark.parametrize("dtype,sizes", [("bf16", (2, 2, 300, 48, 32)), ("bf16", (1, 2, 700, 256, 64)),
                                         ("f32", (1, 2, 333, 30, 16)), ("bf16", (1, 1, 200, 64, 128))])
def test_saved_state_matches_recompute(dtype, sizes):
    """flarepp_mix_save + flarepp_mix_backward_saved: the same Y as flarepp_mix,
    the same Q_dyn and Z as flarepp_mix_debug, and the same gradients as
    flarepp_mix_backward, bit for bit; two encodes fewer."""
    import torch

    require_cuda()
    B, H, N, M, D = sizes
    w = inputs.custom(B, H, N, M, D, dtype=dtype, seed_index=80 + M)
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    dev = [to_dev(x, dtype) for x in (seeds, K, V, dY)]
    Y, saved = flare.flarepp_mix_save(*dev[:3])
    assert saved.numel() == flare.flarepp_saved_bytes(B, H, M, D, dev[1].dtype)
    assert torch.equal(Y, flare.flarepp_mix(*dev[:3]))
    Yd, Qd, Z = flare.flarepp_mix_debug(*dev[:3])
    esz = 2 if dtype == "bf16" else 4
    n = B * H * M * D * esz
    region = (n + 255) // 256 * 256
    assert torch.equal(saved[:n], Qd.reshape(-1).view(torch.uint8))
    assert torch.equal(saved[region:region + n], Z.reshape(-1).view(torch.uint8))
    g_saved = flare.flarepp_mix_backward_saved(*dev, saved)
    launches_saved = flare.flare_last_launch_count()
    g_full = flare.flarepp_mix_backward(*dev)
    # the two recomputed encodes (each with its merge unless it runs one CTA per head)
    assert flare.flare_last_launch_count() == launches_saved + 2 * len(encode_kernels(B, H, N, dtype == "bf16"))
    for a, b in zip(g_saved, g_full):
        assert torch.equal(a, b)
    assert flare.flare_check_status() == (0, 0)
