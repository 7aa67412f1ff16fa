"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Workloads: the five seeded workloads of rank_latent_attention_b200.inputs.
The four smaller ones are compared element by element on every output; the
million-token one (the benchmark's launch configuration) on two full heads
and sampled token rows of Y.  Bars: fp32 path max|err| <= 1e-4; bf16 path
max|err| <= 2e-2 * RMS of the oracle's output, per output tensor.
"""
import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from gpu_common import assert_close, require_cuda, to_dev, to_host
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu

SMALL = ["tiny_f32", "cloud", "mesh2d", "long"]


def _oracle_chain(seeds, K, V):
    return oracle.flarepp_mix(seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64))


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
                   dev=(s_d, K_d, V_d, Qd, Z))
        Qo, Zo, Yo = _oracle_chain(seeds, K, V)
        out[name] = (w, (seeds, K, V), gpu, dict(Q_dyn=Qo, Z=Zo, Y=Yo))
    return out


@pytest.mark.parametrize("name", SMALL)
def test_chain_matches_oracle(small_runs, name):
    w, _, gpu, ref = small_runs[name]
    assert gpu["status"] == (0, 0)
    assert gpu["launches"] == 5  # encode+merge, encode+merge, decode
    for key in ("Q_dyn", "Z", "Y"):
        assert_close(f"{name}.{key}", gpu[key], ref[key], w.dtype)


@pytest.mark.parametrize("name", SMALL)
def test_each_step_matches_oracle(small_runs, name):
    """Each kernel against the oracle step on the same (GPU-produced) inputs."""
    w, (seeds, K, V), gpu, _ = small_runs[name]
    s_d, K_d, V_d, Qd_d, Z_d = gpu["dev"]
    K64, V64 = K.astype(np.float64), V.astype(np.float64)
    Qd_h, Z_h = gpu["Q_dyn"], gpu["Z"]
    # seed encode (Q shared over the batch)
    got = to_host(flare.flare_encode(s_d, K_d, V_d))
    want = np.stack([np.stack([oracle.flare_encode(seeds[h].astype(np.float64), K64[b, h], V64[b, h])
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(f"{name}.seed_encode", got, want, w.dtype)
    # routing encode with the GPU's Q_dyn
    got = to_host(flare.flare_encode(Qd_d, K_d, V_d))
    want = np.stack([np.stack([oracle.flare_encode(Qd_h[b, h], K64[b, h], V64[b, h])
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(f"{name}.routing_encode", got, want, w.dtype)
    # decode with the GPU's Q_dyn and Z
    got = to_host(flare.flare_decode(K_d, Qd_d, Z_d))
    want = np.stack([np.stack([oracle.flare_decode(K64[b, h], Qd_h[b, h], Z_h[b, h])
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close(f"{name}.decode", got, want, w.dtype)
    assert flare.flare_check_status() == (0, 0)


def test_fixed_query_flare(small_runs):
    """FLARE with learned (batch-shared) queries: encode then decode with the same Q."""
    w, (seeds, K, V), gpu, _ = small_runs["long"]
    s_d, K_d, V_d, _, _ = gpu["dev"]
    Z_d = flare.flare_encode(s_d, K_d, V_d)
    Y_d = flare.flare_decode(K_d, s_d, Z_d)
    Zh = to_host(Z_d)
    K64 = K.astype(np.float64)
    want = np.stack([np.stack([oracle.flare_decode(K64[b, h], seeds[h].astype(np.float64), Zh[b, h])
                               for h in range(w.H)]) for b in range(w.B)])
    assert_close("flare.decode_shared_q", to_host(Y_d), want, w.dtype)


def test_million_token_sampled():
    """The benchmark workload (B=1, H=16, N=2^20, M=256, D=64, bf16) in its launch configuration:
    Q_dyn and Z of two full heads and Y on sampled token rows of those heads."""
    torch = require_cuda()
    w = inputs.WORKLOADS["million"]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, w.dtype) for x in (seeds, K, V))
    Y, Qd, Z = flare.flarepp_mix_debug(s_d, K_d, V_d)
    assert flare.flare_check_status() == (0, 0)
    Yh_all, Qdh, Zh = Y, to_host(Qd), to_host(Z)
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([np.arange(8), w.N - 1 - np.arange(200), rng.integers(0, w.N, 4000)]))
    for h in (0, w.H - 1):
        Kh, Vh = K[0, h].astype(np.float64), V[0, h].astype(np.float64)
        Qo = oracle.flare_encode(seeds[h].astype(np.float64), Kh, Vh)
        Zo = oracle.flare_encode(Qo, Kh, Vh)
        assert_close(f"million.h{h}.Q_dyn", Qdh[0, h], Qo, w.dtype)
        assert_close(f"million.h{h}.Z", Zh[0, h], Zo, w.dtype)
        Yo = oracle.flarepp_decode_rows(Kh, Qo, Zo, rows)
        Yg = to_host(Yh_all[0, h][torch.from_numpy(rows).cuda()])
        assert_close(f"million.h{h}.Y_rows", Yg, Yo, w.dtype)
    del K_d, V_d, Y


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
    assert_close("Q_dyn", to_host(Qd), Qo, dtype)
    assert_close("Z", to_host(Z), Zo, dtype)
    assert_close("Y", to_host(Y), Yo, dtype)


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
    assert_close("Q_dyn", to_host(Qd), Qo, w.dtype)
    assert_close("Y", to_host(Y), Yo, w.dtype)


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
