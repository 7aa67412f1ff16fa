"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Workloads: the five seeded workloads of rank_latent_attention_b200.inputs.
The four smaller ones are compared element by element on every output; the
million-token one (the benchmark's launch configuration) on two full heads
and sampled token rows of Y.

Bars (tests/gpu_common.py): the stated bar (fp32 1e-4 absolute; bf16 inputs
2e-2 x RMS of the oracle output) holds for the fp32 path everywhere, and for
the split-precision tensor-core mode (FLARE_BF16_F32OUT: bf16 inputs, hi/lo
bf16 operand pairs, fp32 Q_dyn, Z and Y) on every bf16 workload.  The bf16
tensor-core path (everything stored in bf16) is held to the stated bar on
the Gaussian workloads and to the per-head bf16-storage bar everywhere: on
mesh2d and long the bf16 storage of the chain alone, with exact arithmetic
otherwise, exceeds the stated bar (tests/test_tolerance_analysis.py).
"""
import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from gpu_common import assert_bf16_storage, assert_stated, mix_kernels, require_cuda, to_dev, to_host
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu

SMALL = ["tiny_f32", "cloud", "mesh2d", "long"]
# workloads where three chained bf16 SDPA calls (Q_dyn, Z and Y stored as
# bf16, exact arithmetic otherwise) fit the stated bar; the CPU tests in
# test_tolerance_analysis.py show mesh2d and long do not
STATED_HOLDS_FOR_BF16 = {"cloud", "million"}
# the kernels one flarepp_mix call launches on the tensor cores when each
# encode runs more than one CTA per head (one: no merges, see mix_kernels)
TC_CHAIN = ["encode_tc", "lse_merge", "encode_tc", "lse_merge", "decode_tc"]


def _oracle_chain(seeds, K, V):
    return oracle.flarepp_mix(seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64))


def _check_outputs(name, w, got, ref, V):
    """got / ref: dicts with Q_dyn, Z, Y; V the inputs [B, H, N, D]."""
    if w.dtype == "f32":
        for key in ("Q_dyn", "Z", "Y"):
            assert_stated(f"{name}.{key}", got[key], ref[key], "f32")
        return
    assert_bf16_storage(f"{name}.Q_dyn", got["Q_dyn"], ref["Q_dyn"], V, 2)
    assert_bf16_storage(f"{name}.Z", got["Z"], ref["Z"], V, 2)
    assert_bf16_storage(f"{name}.Y", got["Y"], ref["Y"], ref["Z"], 16)
    if name in STATED_HOLDS_FOR_BF16:
        assert_stated(f"{name}.Y", got["Y"], ref["Y"], "bf16")


@pytest.fixture(scope="module")
def small_runs():
    """Inputs, GPU outputs (chained, with intermediates) and oracle outputs per small workload."""
    require_cuda()
    out = {}
    for name in SMALL:
        w = inputs.WORKLOADS[name]
        seeds, K, V = inputs.make_inputs(w)
        s_d, K_d, V_d = (to_dev(x, w.dtype) for x in (seeds, K, V))
        Y, Qd, Z = flare.flarepp_mix_debug(s_d, K_d, V_d)
        launches = flare.flare_last_launch_count()
        st = flare.flare_check_status()
        gpu = dict(Y=to_host(Y), Q_dyn=to_host(Qd), Z=to_host(Z), launches=launches, status=st,
                   dev=(s_d, K_d, V_d, Qd, Z),
                   chain=mix_kernels(w.B, w.H, w.N, w.dtype != "f32"))
        Qo, Zo, Yo = _oracle_chain(seeds, K, V)
        out[name] = (w, (seeds, K, V), gpu, dict(Q_dyn=Qo, Z=Zo, Y=Yo))
    return out


@pytest.mark.parametrize("name", SMALL)
def test_chain_matches_oracle(small_runs, name):
    w, (_, _, V), gpu, ref = small_runs[name]
    assert gpu["status"] == (0, 0)
    assert gpu["launches"] == len(gpu["chain"])  # encode (+ merge), encode (+ merge), decode
    _check_outputs(name, w, gpu, ref, V.astype(np.float64))


def _split_precision(s_d, K_d, V_d):
    """flarepp_mix_debug in the split-precision mode; returns (Y, Q_dyn, Z) and the kernels it launched."""
    import torch
    flare.flare_profile_begin(16)
    try:
        Y, Qd, Z = flare.flarepp_mix_debug(s_d, K_d, V_d, out_dtype=torch.float32)
    finally:
        kernels = [k for k, _ in flare.flare_profile_end()]
    assert flare.flare_check_status() == (0, 0)
    assert Y.dtype == Qd.dtype == Z.dtype == torch.float32
    return Y, Qd, Z, kernels


@pytest.mark.parametrize("name", ["cloud", "mesh2d", "long"])
def test_split_precision_meets_stated_bar(small_runs, name):
    """bf16 seeds/K/V; every rounded MMA operand (P, Q_dyn, Z) as a hi/lo bf16
    pair on the tensor cores, fp32 Q_dyn, Z and Y: the stated 2e-2 x RMS bar
    on every bf16 workload, through the tcgen05 kernels."""
    w, _, gpu, ref = small_runs[name]
    s_d, K_d, V_d, _, _ = gpu["dev"]
    Y, Qd, Z, kernels = _split_precision(s_d, K_d, V_d)
    assert kernels == mix_kernels(w.B, w.H, w.N)
    for key, val in (("Q_dyn", Qd), ("Z", Z), ("Y", Y)):
        assert_stated(f"{name}.split.{key}", to_host(val), ref[key], "bf16")


SPLIT_EDGE = [
    # (B, H, N, M, D): tensor cores (M % 16 == 0, D <= 64), ragged and one-token heads
    (1, 1, 1, 16, 16),
    (1, 2, 2, 32, 64),
    (2, 1, 127, 48, 32),
    (1, 1, 129, 144, 64),
    (1, 3, 257, 256, 16),
    (2, 2, 1000, 256, 32),
    (1, 2, 5000, 128, 64),
    # CUDA-core kernels of the same mode: M % 16 != 0, D = 128
    (1, 2, 300, 33, 32),
    (1, 1, 700, 256, 128),
]


@pytest.mark.parametrize("B,H,N,M,D", SPLIT_EDGE)
def test_split_precision_edge_shapes(B, H, N, M, D):
    require_cuda()
    w = inputs.custom(B, H, N, M, D, dtype="bf16", scale=0.6)
    seeds, K, V = inputs.make_inputs(w)
    Y, Qd, Z, kernels = _split_precision(*(to_dev(x, "bf16") for x in (seeds, K, V)))
    tc = M % 16 == 0 and D <= 64
    assert kernels == mix_kernels(B, H, N, tc)
    Qo, Zo, Yo = _oracle_chain(seeds, K, V)
    for key, got, want in (("Q_dyn", Qd, Qo), ("Z", Z, Zo), ("Y", Y, Yo)):
        assert_stated(f"split{(B, H, N, M, D)}.{key}", to_host(got), want, "bf16")


@pytest.mark.parametrize("splits", [1, 2, 3, 1000])
def test_split_precision_split_counts(splits):
    require_cuda()
    w = inputs.WORKLOADS["long"]
    seeds, K, V = inputs.make_inputs(w)
    seeds, K, V = seeds, K[:2], V[:2]  # two batch elements keep the oracle quick
    dev = [to_dev(x, w.dtype) for x in (seeds, K, V)]
    old = flare.flare_set_split_override(splits)
    try:
        Y, Qd, Z, kernels = _split_precision(*dev)
        chain = mix_kernels(2, w.H, w.N)
    finally:
        flare.flare_set_split_override(old)
    assert kernels == chain
    assert (splits == 1) == ("lse_merge" not in chain)
    Qo, Zo, Yo = _oracle_chain(seeds, K, V)
    for key, got, want in (("Q_dyn", Qd, Qo), ("Z", Z, Zo), ("Y", Y, Yo)):
        assert_stated(f"long[:2] splits={splits}.{key}", to_host(got), want, "bf16")


@pytest.mark.parametrize("M,D", [(256, 64), (64, 32)])
def test_split_precision_reference_far_behind(M, D):
    """The climbing logits of test_encode_reference_far_behind as the seeds of
    the split-precision chain: the seed encode's skip-max fallback with hi/lo P
    (one CTA per head), checked on Q_dyn and on the chained Y."""
    require_cuda()
    H, N = 2, 64 * 70 + 37
    Q, K, V = inputs.make_climbing(H, N, M, D, jump_tile=50)
    old = flare.flare_set_split_override(1)
    try:
        Y, Qd, Z, kernels = _split_precision(*(to_dev(x, "bf16") for x in (Q, K, V)))
    finally:
        flare.flare_set_split_override(old)
    assert kernels == ["encode_tc", "encode_tc", "decode_tc"]  # one CTA per head: no merges
    Qo, Zo, Yo = _oracle_chain(Q, K, V)
    for key, got, want in (("Q_dyn", Qd, Qo), ("Z", Z, Zo), ("Y", Y, Yo)):
        assert_stated(f"climb-split{(M, D)}.{key}", to_host(got), want, "bf16")


@pytest.mark.parametrize("name", SMALL)
def test_each_step_matches_oracle(small_runs, name):
    """Each kernel against the oracle step on the same (GPU-produced) inputs."""
    w, (seeds, K, V), gpu, _ = small_runs[name]
    s_d, K_d, V_d, Qd_d, Z_d = gpu["dev"]
    K64, V64 = K.astype(np.float64), V.astype(np.float64)
    Qd_h, Z_h = gpu["Q_dyn"], gpu["Z"]

    def per_head(fn):
        return np.stack([np.stack([fn(b, h) for h in range(w.H)]) for b in range(w.B)])

    steps = [
        ("seed_encode", flare.flare_encode(s_d, K_d, V_d),
         per_head(lambda b, h: oracle.flare_encode(seeds[h].astype(np.float64), K64[b, h], V64[b, h])), V64, 2),
        ("routing_encode", flare.flare_encode(Qd_d, K_d, V_d),
         per_head(lambda b, h: oracle.flare_encode(Qd_h[b, h], K64[b, h], V64[b, h])), V64, 2),
    ]
    dec = per_head(lambda b, h: oracle.flare_decode(K64[b, h], Qd_h[b, h], Z_h[b, h]))
    steps.append(("decode", flare.flare_decode(K_d, Qd_d, Z_d), dec, Z_h, 4))
    for label, got_d, want, rows, c in steps:
        got = to_host(got_d)
        if w.dtype == "f32":
            assert_stated(f"{name}.{label}", got, want, "f32")
        else:
            assert_bf16_storage(f"{name}.{label}", got, want, rows, c)
    assert flare.flare_check_status() == (0, 0)


def test_fixed_query_flare(small_runs):
    """FLARE with learned (batch-shared) queries: encode then decode with the same Q."""
    w, (seeds, K, V), gpu, _ = small_runs["cloud"]
    s_d, K_d, V_d, _, _ = gpu["dev"]
    Z_d = flare.flare_encode(s_d, K_d, V_d)
    Y_d = flare.flare_decode(K_d, s_d, Z_d)
    K64, V64 = K.astype(np.float64), V.astype(np.float64)
    Zo = np.stack([np.stack([oracle.flare_encode(seeds[h].astype(np.float64), K64[b, h], V64[b, h])
                             for h in range(w.H)]) for b in range(w.B)])
    Yo = np.stack([np.stack([oracle.flare_decode(K64[b, h], seeds[h].astype(np.float64), Zo[b, h])
                             for h in range(w.H)]) for b in range(w.B)])
    assert_stated("flare.Z", to_host(Z_d), Zo, "bf16")
    assert_stated("flare.Y", to_host(Y_d), Yo, "bf16")


def test_million_token_sampled():
    """The benchmark workload (B=1, H=16, N=2^20, M=256, D=64, bf16) in its launch configuration:
    Q_dyn and Z of two full heads and Y on sampled token rows of those heads (RMS over the sample)."""
    torch = require_cuda()
    w = inputs.WORKLOADS["million"]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, w.dtype) for x in (seeds, K, V))
    Y, Qd, Z = flare.flarepp_mix_debug(s_d, K_d, V_d)
    assert flare.flare_check_status() == (0, 0)
    Qdh, Zh = to_host(Qd), to_host(Z)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([np.arange(8), w.N - 1 - np.arange(200), rng.integers(0, w.N, 4000)]))
    heads = (0, w.H - 1)
    Qo, Zo, Yo, Yg = [], [], [], []
    for h in heads:
        Kh, Vh = K[0, h].astype(np.float64), V[0, h].astype(np.float64)
        q = oracle.flare_encode(seeds[h].astype(np.float64), Kh, Vh)
        z = oracle.flare_encode(q, Kh, Vh)
        Qo.append(q)
        Zo.append(z)
        Yo.append(oracle.flarepp_decode_rows(Kh, q, z, rows))
        Yg.append(to_host(Y[0, h][torch.from_numpy(rows).cuda()]))
    Qo, Zo, Yo, Yg = (np.stack(x)[None] for x in (Qo, Zo, Yo, Yg))
    for key, got, want in (("Q_dyn", Qdh[:, list(heads)], Qo), ("Z", Zh[:, list(heads)], Zo), ("Y_rows", Yg, Yo)):
        assert_stated(f"million.{key}", got, want, "bf16")
    assert_bf16_storage("million.Y_rows", Yg, Yo, Zo, 16)
    # the same workload in the split-precision mode, same checks at the stated bar
    del Y, Qd, Z
    Y, Qd, Z, kernels = _split_precision(s_d, K_d, V_d)
    assert kernels == TC_CHAIN  # 37 CTAs per head
    Yg = np.stack([to_host(Y[0, h][torch.from_numpy(rows).cuda()]) for h in heads])[None]
    for key, got, want in (("Q_dyn", to_host(Qd)[:, list(heads)], Qo), ("Z", to_host(Z)[:, list(heads)], Zo),
                           ("Y_rows", Yg, Yo)):
        assert_stated(f"million.split.{key}", got, want, "bf16")


EDGE = [
    # (B, H, N, M, D, dtype)
    (1, 1, 1, 16, 16, "bf16"),
    (1, 2, 2, 32, 64, "bf16"),
    (2, 1, 127, 48, 32, "bf16"),
    (1, 1, 128, 128, 128, "bf16"),
    (1, 1, 129, 144, 64, "bf16"),
    (1, 3, 257, 256, 16, "bf16"),
    (2, 2, 1000, 256, 128, "bf16"),
    (1, 1, 1, 1, 16, "f32"),
    (1, 2, 129, 33, 64, "f32"),
    (2, 1, 300, 256, 128, "f32"),
    (1, 1, 5000, 200, 32, "f32"),
]


@pytest.mark.parametrize("B,H,N,M,D,dtype", EDGE)
def test_edge_shapes(B, H, N, M, D, dtype):
    require_cuda()
    w = inputs.custom(B, H, N, M, D, dtype=dtype, scale=0.6)
    seeds, K, V = inputs.make_inputs(w)
    Y, Qd, Z = flare.flarepp_mix_debug(*(to_dev(x, dtype) for x in (seeds, K, V)))
    assert flare.flare_check_status() == (0, 0)
    Qo, Zo, Yo = _oracle_chain(seeds, K, V)
    _check_outputs(f"edge{(B, H, N, M, D)}", w, dict(Q_dyn=to_host(Qd), Z=to_host(Z), Y=to_host(Y)),
                   dict(Q_dyn=Qo, Z=Zo, Y=Yo), V.astype(np.float64))


@pytest.mark.parametrize("splits", [1, 2, 3, 1000])
@pytest.mark.parametrize("name", ["cloud", "tiny_f32"])
def test_split_counts_agree(name, splits):
    """The exact log-sum-exp merge makes the result independent of how tokens are split."""
    require_cuda()
    w = inputs.WORKLOADS[name]
    seeds, K, V = inputs.make_inputs(w)
    dev = [to_dev(x, w.dtype) for x in (seeds, K, V)]
    old = flare.flare_set_split_override(splits)
    try:
        Y, Qd, Z = flare.flarepp_mix_debug(*dev)
        assert flare.flare_check_status() == (0, 0)
    finally:
        flare.flare_set_split_override(old)
    Qo, Zo, Yo = _oracle_chain(seeds, K, V)
    assert_stated("Q_dyn", to_host(Qd), Qo, w.dtype)
    assert_stated("Y", to_host(Y), Yo, w.dtype)


@pytest.mark.parametrize("M,D", [(256, 64), (64, 64), (144, 32), (256, 16), (128, 128)])
@pytest.mark.parametrize("splits", [1, 0])
def test_encode_reference_far_behind(M, D, splits):
    """The encode keeps each row's running reference until a tile's sum of
    2^(x log2e - reference) leaves [0, 2^32]; then it takes the tile's max.
    Logits that climb about 6 per 64-token tile (inputs.make_climbing: a
    reference falls 2^32 behind within a few tiles) and one tile that jumps
    120 higher, past the fp32 range of 2^(x - reference), exercise that
    fallback: with one CTA per head every tile after the first goes through
    it; and with the default split count.  D = 128 always takes the max."""
    require_cuda()
    H, N = 2, 64 * 70 + 37
    Q, K, V = inputs.make_climbing(H, N, M, D, jump_tile=50)
    old = flare.flare_set_split_override(splits)
    try:
        Z = flare.flare_encode(to_dev(Q, "bf16"), to_dev(K, "bf16"), to_dev(V, "bf16"))
        assert flare.flare_check_status() == (0, 0)
    finally:
        flare.flare_set_split_override(old)
    Zo = np.stack([oracle.flare_encode(Q[h].astype(np.float64), K[0, h].astype(np.float64),
                                       V[0, h].astype(np.float64)) for h in range(H)])[None]
    assert_bf16_storage(f"climb{(M, D, splits)}.Z", to_host(Z), Zo, V.astype(np.float64), 2)
    # the jump tile dominates: Z is a convex mix of its values
    jump = V[0, :, 50 * 64:51 * 64].astype(np.float64)
    assert np.all(to_host(Z) <= jump.max(axis=1)[None, :, None, :] + 1e-2)
    assert np.all(to_host(Z) >= jump.min(axis=1)[None, :, None, :] - 1e-2)


def test_caller_workspace_and_stream():
    """Caller-provided workspace on a side stream gives the same result as the internal one."""
    torch = require_cuda()
    w = inputs.WORKLOADS["mesh2d"]
    seeds, K, V = inputs.make_inputs(w)
    dev = [to_dev(x, w.dtype) for x in (seeds, K, V)]
    ref = flare.flarepp_mix(*dev)
    nbytes = flare.flarepp_workspace_size(w.B, w.H, w.N, w.M, w.D, 1)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        got = flare.flarepp_mix(*dev, workspace=ws, stream=s)
    s.synchronize()
    assert torch.equal(got, ref)
    too_small = torch.empty(nbytes - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(flare.FlareError):
        flare.flarepp_mix(*dev, workspace=too_small)


def test_cpu_tensor_rejected():
    torch = require_cuda()
    x = torch.zeros(1, 1, 8, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        flare.flarepp_mix(torch.zeros(1, 16, 16, dtype=torch.bfloat16), x, x)
