"""Out-of-bounds writes, without compute-sanitizer (closed on this pool):
every output and workspace buffer sits between 4 KB guard bands of 0xFF
bytes (NaN in bf16 and fp32), and after each entry point ran the bands must
be untouched and the inputs unchanged.  Shapes cover ragged token tails,
latent counts that are not multiples of the tiles, every D and both dtypes.
"""
import pytest

import rank_latent_attention_b200 as flare
from gpu_common import require_cuda, to_dev
from rank_latent_attention_b200 import context_parallel as cp
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu

GUARD = 4096


class Guarded:
    """Tensors carved out of one buffer, each between guard bands."""

    def __init__(self):
        import torch

        self.torch = torch
        self.items = []

    def tensor(self, shape, dtype):
        torch = self.torch
        n = 1
        for x in shape:
            n *= x
        nbytes = n * torch.empty((), dtype=dtype).element_size()
        inner = (nbytes + 255) // 256 * 256
        buf = torch.full((2 * GUARD + inner,), 0xFF, dtype=torch.uint8, device="cuda")
        view = buf[GUARD:GUARD + nbytes].view(dtype).view(shape)
        self.items.append((buf, nbytes))
        return view

    def check(self, label):
        for k, (buf, nbytes) in enumerate(self.items):
            head = buf[:GUARD]
            tail = buf[GUARD + nbytes:]
            assert bool((head == 0xFF).all()), f"{label}: buffer {k} written below its start"
            assert bool((tail == 0xFF).all()), f"{label}: buffer {k} written past its end"


CASES = [  # B, H, N, M, D, dtype
    (2, 3, 333, 48, 32, "bf16"),
    (1, 2, 129, 256, 64, "bf16"),
    (1, 2, 257, 16, 16, "bf16"),
    (1, 1, 200, 144, 128, "bf16"),
    (2, 2, 97, 30, 16, "f32"),
]


@pytest.mark.parametrize("B,H,N,M,D,dtype", CASES)
def test_forward_and_backward_stay_in_bounds(B, H, N, M, D, dtype):
    torch = require_cuda()
    w = inputs.custom(B, H, N, M, D, dtype=dtype, seed_index=97)
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    s_d, K_d, V_d, dY_d = (to_dev(x, dtype) for x in (seeds, K, V, dY))
    originals = [x.clone() for x in (s_d, K_d, V_d, dY_d)]
    tdt = s_d.dtype
    code = flare.BF16 if dtype == "bf16" else flare.F32
    g = Guarded()

    # forward with intermediates, caller workspace exactly sized
    Y, Qd, Z = g.tensor((B, H, N, D), tdt), g.tensor((B, H, M, D), tdt), g.tensor((B, H, M, D), tdt)
    ws = g.tensor((flare.flarepp_workspace_size(B, H, N, M, D, code),), torch.uint8)
    flare.flarepp_mix_debug(s_d, K_d, V_d, Y=Y, Q_dyn=Qd, Z=Z, workspace=ws)
    # saved state and both backward forms
    saved = g.tensor((flare.flarepp_saved_bytes(B, H, M, D, code),), torch.uint8)
    flare.flarepp_mix_save(s_d, K_d, V_d, Y, saved)
    grads = (g.tensor((H, M, D), tdt), g.tensor((B, H, N, D), tdt), g.tensor((B, H, N, D), tdt))
    wsb = g.tensor((flare.flarepp_mix_backward_workspace_size(B, H, N, M, D, code),), torch.uint8)
    flare.flarepp_mix_backward(s_d, K_d, V_d, dY_d, *grads, workspace=wsb)
    flare.flarepp_mix_backward_saved(s_d, K_d, V_d, dY_d, saved, *grads, workspace=wsb)
    # a token shard's encode and the combine
    O, lse = g.tensor((B, H, M, D), torch.float32), g.tensor((B, H, M), torch.float32)
    wse = g.tensor((max(1, flare.flare_encode_lse_workspace_size(B, H, N, M, D, code)),), torch.uint8)
    flare.flare_encode_lse(s_d, K_d, V_d, O=O, lse=lse, workspace=wse)
    out, L = g.tensor((B, H, M, D), tdt), g.tensor((B, H, M), torch.float32)
    flare.flare_lse_combine(O[None].contiguous(), lse[None].contiguous(), out=out, lse_out=L)
    # one phase cycle of the sharded backward on the whole cloud
    lib = flare.lib()
    exch = g.tensor((lib.flarepp_backward_shard_exchange_floats(B, H, M, D),), torch.float32)
    wss = g.tensor((lib.flarepp_backward_shard_workspace_size(B, H, N, M, D, code),), torch.uint8)
    for phase in range(4):
        flare.flarepp_mix_backward_shard(phase, s_d, K_d, V_d, dY_d, saved, exch, *grads, wss)
    assert flare.flare_check_status() == (0, 0)
    torch.cuda.synchronize()
    g.check(f"{B}x{H}x{N}x{M}x{D}_{dtype}")
    for a, b in zip((s_d, K_d, V_d, dY_d), originals):
        assert torch.equal(a, b), "an input was written"
