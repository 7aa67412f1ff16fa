"""flarepp_mix_host: the mixer with seeds, K, V and Y in host memory, heads
streamed through the GPU with the copies overlapping the compute.

Results against the oracle at the bars of the device path (the host path runs
the same kernels, one head at a time), in page-locked and pageable memory,
for the bf16, fp32 and bf16-in / fp32-out modes; a device pointer where host
memory is expected is rejected before any work.
"""
import ctypes

import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from rank_latent_attention_b200 import inputs
from gpu_common import assert_stated, require_cuda

pytestmark = pytest.mark.gpu


def _host(arr, dtype, pin):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    t = t.to(torch.bfloat16) if dtype == "bf16" else t
    return t.pin_memory() if pin else t


def _oracle_Y(seeds, K, V):
    return oracle.flarepp_mix(seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64))[2]


@pytest.mark.parametrize("name,pin", [("cloud", True), ("tiny_f32", False)])
def test_host_mix_matches_oracle(name, pin):
    torch = require_cuda()
    w = inputs.WORKLOADS[name]
    seeds, K, V = inputs.make_inputs(w)
    Y = flare.flarepp_mix_host(*(_host(x, w.dtype, pin) for x in (seeds, K, V)))
    torch.cuda.current_stream().synchronize()
    assert flare.flare_check_status() == (0, 0)
    assert flare.flare_last_launch_count() == 5 * w.B * w.H  # one mix per (b, h)
    assert_stated(f"{name}.Y", Y.float().numpy().astype(np.float64), _oracle_Y(seeds, K, V), w.dtype)


def test_host_mix_fp32_output_and_workspace():
    torch = require_cuda()
    w = inputs.WORKLOADS["mesh2d"]
    seeds, K, V = inputs.make_inputs(w)
    sh, Kh, Vh = (_host(x, "bf16", True) for x in (seeds, K, V))
    nbytes = flare.lib().flarepp_mix_host_workspace_size(w.B, w.H, w.N, w.M, w.D, flare.BF16_F32OUT)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    Y1 = flare.flarepp_mix_host(sh, Kh, Vh, out_dtype=torch.float32, workspace=ws)
    Y2 = flare.flarepp_mix_host(sh, Kh, Vh, out_dtype=torch.float32, workspace=ws)
    torch.cuda.current_stream().synchronize()
    assert flare.flare_check_status() == (0, 0)
    assert Y1.dtype == torch.float32 and torch.equal(Y1, Y2)
    # same kernels, same per-head split as the device path run one head at a time
    Yd = torch.stack([torch.stack([flare.flarepp_mix(sh[h:h + 1].cuda(), Kh[b:b + 1, h:h + 1].cuda(),
                                                     Vh[b:b + 1, h:h + 1].cuda(), out_dtype=torch.float32)[0, 0]
                                   for h in range(w.H)]) for b in range(w.B)])
    assert torch.equal(Y1, Yd.cpu())


def test_device_pointer_rejected():
    torch = require_cuda()
    w = inputs.custom(1, 1, 64, 16, 16, dtype="bf16")
    seeds, K, V = inputs.make_inputs(w)
    sh, Kh, Vh = (_host(x, "bf16", True) for x in (seeds, K, V))
    Yd = torch.empty((1, 1, 64, 16), dtype=torch.bfloat16, device="cuda")
    rc = flare.lib().flarepp_mix_host(sh.data_ptr(), Kh.data_ptr(), Vh.data_ptr(), Yd.data_ptr(), 1, 1, 64, 16, 16,
                                      flare.BF16, None, 0, None)
    assert rc == 1  # FLARE_ERR_INVALID_ARG
