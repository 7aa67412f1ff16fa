"""flare_encode_noalloc against flare_encode (GPU, through the C ABI).

flare_encode_noalloc serves callers that may not allocate device memory: it
keeps the encode's scratch in a fixed array inside the library instead of a
workspace.  Its results must equal those of flare_encode, which takes (or
allocates) a workspace, on calls made one after another with different sizes
(the array keeps the previous call's contents), and sizes whose scratch does
not fit must be refused before anything runs.  This file is collected last
so that a stop at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import rank_latent_attention_b200 as flare
from gpu_common import require_cuda, to_dev, to_host
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu

_vp = ctypes.c_void_p


def _noalloc():
    fn = flare.lib().flare_encode_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [_vp, ctypes.c_int, _vp, _vp, _vp, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                   ctypes.c_int, ctypes.c_int, _vp]
    return fn


def _call(fn, Q, K, V, Z, dtype_code):
    import torch
    B, H, N, D = K.shape
    M = Q.shape[-2]
    q_batched = 1 if Q.dim() == 4 else 0
    return fn(_vp(Q.data_ptr()), q_batched, _vp(K.data_ptr()), _vp(V.data_ptr()), _vp(Z.data_ptr()),
              B, H, N, M, D, dtype_code, _vp(torch.cuda.current_stream().cuda_stream))


def _workload(name):
    # "m256": two latent halves (M = 256), so the encode's two slots each fold
    # their accumulators into the fixed array; 74 partials per head
    return inputs.custom(1, 2, 8192, 256, 32, "bf16") if name == "m256" else inputs.WORKLOADS[name]


@pytest.mark.parametrize("sequence", [("cloud", "mesh2d"), ("tiny_f32", "tiny_f32"), ("mesh2d", "cloud"),
                                      ("m256", "mesh2d", "m256"), ("mesh2d", "m256", "cloud")])
def test_noalloc_matches_encode_on_consecutive_calls(sequence):
    """Same kernels, same split count: the results must be the same bits."""
    torch = require_cuda()
    fn = _noalloc()
    for name in sequence:
        w = _workload(name)
        assert flare.flare_encode_workspace_size(w.B, w.H, w.N, w.M, w.D, 1 if w.dtype == "bf16" else 0) \
            <= (16 << 20)
        seeds, K, V = inputs.make_inputs(w)
        s_d, K_d, V_d = (to_dev(x, w.dtype) for x in (seeds, K, V))
        want = flare.flare_encode(s_d, K_d, V_d)
        got = torch.full_like(want, float("nan"))
        code = 1 if w.dtype == "bf16" else 0
        assert _call(fn, s_d, K_d, V_d, got, code) == 0
        assert flare.flare_check_status() == (0, 0)
        assert torch.equal(got, want), (name, float(np.max(np.abs(to_host(got) - to_host(want)))))


def test_noalloc_refuses_scratch_beyond_its_array():
    torch = require_cuda()
    fn = _noalloc()
    B, H, N, M, D = 1, 16, 1 << 20, 256, 64  # partials need ~39 MiB
    assert flare.flare_encode_workspace_size(B, H, N, M, D, 1) > (16 << 20)
    K = torch.zeros((B, H, N, D), dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros((H, M, D), dtype=torch.bfloat16, device="cuda")
    Z = torch.zeros((B, H, M, D), dtype=torch.bfloat16, device="cuda")
    assert _call(fn, Q, K, K, Z, 1) == 2  # FLARE_ERR_UNSUPPORTED, nothing enqueued
    assert torch.count_nonzero(Z).item() == 0
