"""GPU parity of the token-sharded encode (flare_encode_lse, flare_lse_combine)
and of the context-parallel mixer built on them, against the fp64 oracle
("FLARE++" page, "Contributions Clés", context-parallelism item).

Ranks are emulated on the one GPU one after another: each rank's shard encode
writes its row of the gathered buffer, which is what the all-gather returns;
no kernel waits on another.  A world-size-1 NCCL process group runs the real
collective path.

Bars: O and the combined outputs as the encode's (tests/gpu_common.py, per
head 2e-2 RMS + 2 x 2^-9 max|V| for bf16, 1e-4 for fp32); Y as the decode's
(c = 16).  lse: the shard's exp sum carries at most ~1e-4 relative error
(the polynomial share's 7.5e-5 bound, MUFU ex2's few ulp) and the logits are
fp32 sums of exact bf16 products, so |lse - oracle| <= 5e-4 (bf16) and 1e-4
(fp32 SIMT, exp2f).
"""
import datetime

import numpy as np
import pytest

import oracle
import rank_latent_attention_b200 as flare
from gpu_common import (assert_backward_bar, assert_bf16_storage, assert_stated, encode_kernels, require_cuda, to_dev,
                        to_host)
from rank_latent_attention_b200 import context_parallel as cp
from rank_latent_attention_b200 import inputs

pytestmark = pytest.mark.gpu

LSE_TOL = {"bf16": 5e-4, "f32": 1e-4}


def _per_head(B, H, fn):
    return np.stack([np.stack([fn(b, h) for h in range(H)]) for b in range(B)])


def _emulate(s_d, K_d, V_d, R):
    """The context-parallel mixer with R ranks emulated in turn on this GPU."""
    import torch

    B, H, N, D = K_d.shape
    M = s_d.shape[-2]
    ops = cp.LibraryOps()
    recv = torch.empty((R, cp.exchange_floats(B, H, M, D)), dtype=torch.float32, device="cuda")
    shards = [(cp.shard_tokens(K_d, R, r), cp.shard_tokens(V_d, R, r)) for r in range(R)]

    def encode(Q):
        for r, (Kr, Vr) in enumerate(shards):
            ops.encode_lse(Q, Kr, Vr, recv[r])
        return ops.combine(recv, B, H, M, D, K_d.dtype)

    Qd = encode(s_d)
    Z = encode(Qd)
    Y = torch.cat([ops.decode(Kr, Qd, Z) for Kr, _ in shards], dim=2)
    return Y, Qd, Z


def _check(name, w, got, ref, V64):
    if w.dtype == "f32":
        for key in ("Q_dyn", "Z", "Y"):
            assert_stated(f"{name}.{key}", got[key], ref[key], "f32")
        return
    assert_bf16_storage(f"{name}.Q_dyn", got["Q_dyn"], ref["Q_dyn"], V64, 2)
    assert_bf16_storage(f"{name}.Z", got["Z"], ref["Z"], V64, 2)
    assert_bf16_storage(f"{name}.Y", got["Y"], ref["Y"], ref["Z"], 16)


@pytest.mark.parametrize("name,R", [("tiny_f32", 3), ("cloud", 4), ("mesh2d", 3), ("long", 2)])
def test_shard_encode_lse(name, R):
    """Each shard's (O, lse) against the oracle's encode_shard."""
    require_cuda()
    w = inputs.WORKLOADS[name]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, w.dtype) for x in (seeds, K, V))
    K64, V64, S64 = K.astype(np.float64), V.astype(np.float64), seeds.astype(np.float64)
    for r in range(R):
        a, b = cp.token_range(w.N, R, r)
        O, lse = flare.flare_encode_lse(s_d, cp.shard_tokens(K_d, R, r), cp.shard_tokens(V_d, R, r))
        # the shard's encode (+ its merge unless it runs one CTA per head)
        assert flare.flare_last_launch_count() == len(encode_kernels(w.B, w.H, b - a, w.dtype != "f32"))
        ref = [[oracle.encode_shard(S64[h], K64[bb, h, a:b], V64[bb, h, a:b]) for h in range(w.H)]
               for bb in range(w.B)]
        Oo = np.array([[x[0] for x in row] for row in ref])
        Lo = np.array([[x[1] for x in row] for row in ref])
        if w.dtype == "f32":
            assert_stated(f"{name}.O[{r}]", to_host(O), Oo, "f32")
        else:
            assert_bf16_storage(f"{name}.O[{r}]", to_host(O), Oo, V64[:, :, a:b], 2)
        err = float(np.max(np.abs(to_host(lse) - Lo)))
        assert err <= LSE_TOL[w.dtype], (name, r, err)
    assert flare.flare_check_status() == (0, 0)


@pytest.mark.parametrize("name,R", [("tiny_f32", 2), ("cloud", 3), ("mesh2d", 4), ("long", 5)])
def test_emulated_ranks_match_oracle(name, R):
    require_cuda()
    w = inputs.WORKLOADS[name]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, w.dtype) for x in (seeds, K, V))
    Y, Qd, Z = _emulate(s_d, K_d, V_d, R)
    assert flare.flare_check_status() == (0, 0)
    Qo, Zo, Yo = oracle.flarepp_mix(seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64))
    got = dict(Q_dyn=to_host(Qd), Z=to_host(Z), Y=to_host(Y))
    _check(f"{name}.cp{R}", w, got, dict(Q_dyn=Qo, Z=Zo, Y=Yo), V.astype(np.float64))


def test_empty_shards():
    """3 tokens over 5 ranks: two ranks hold none; N = 0 gives O = 0, lse = -inf exactly."""
    import torch

    require_cuda()
    w = inputs.custom(2, 2, 3, 16, 16, dtype="bf16", seed_index=61)
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, "bf16") for x in (seeds, K, V))
    O, lse = flare.flare_encode_lse(s_d, K_d[:, :, :0], V_d[:, :, :0])
    assert flare.flare_last_launch_count() == 1
    assert torch.all(O == 0) and torch.all(torch.isneginf(lse))
    Y, Qd, Z = _emulate(s_d, K_d, V_d, 5)
    assert flare.flare_check_status() == (0, 0)
    Qo, Zo, Yo = oracle.flarepp_mix(seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64))
    _check("empty_shards", w, dict(Q_dyn=to_host(Qd), Z=to_host(Z), Y=to_host(Y)),
           dict(Q_dyn=Qo, Z=Zo, Y=Yo), V.astype(np.float64))
    # every shard empty: out = 0, L = -inf
    Oe = torch.zeros((3, 2, 2, 16, 16), dtype=torch.float32, device="cuda")
    Le = torch.full((3, 2, 2, 16), float("-inf"), device="cuda")
    L = torch.empty((2, 2, 16), device="cuda")
    out = flare.flare_lse_combine(Oe, Le, lse_out=L, dtype=torch.float32)
    assert torch.all(out == 0) and torch.all(torch.isneginf(L))


def test_combine_layouts_and_lse():
    """Dense stacks and the packed all-gather rows give the same bits; the
    combined lse is the log-sum-exp over all tokens."""
    import torch

    require_cuda()
    w = inputs.WORKLOADS["cloud"]
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, "bf16") for x in (seeds, K, V))
    R = 3
    parts = [flare.flare_encode_lse(s_d, cp.shard_tokens(K_d, R, r), cp.shard_tokens(V_d, R, r)) for r in range(R)]
    O_st = torch.stack([p[0] for p in parts])
    L_st = torch.stack([p[1] for p in parts])
    L1 = torch.empty_like(parts[0][1])
    dense = flare.flare_lse_combine(O_st, L_st, lse_out=L1)
    assert flare.flare_last_launch_count() == 1
    packed = torch.cat([torch.cat([p[0].reshape(-1), p[1].reshape(-1)]) for p in parts])
    n = O_st[0].numel()
    L2 = torch.empty_like(L1)
    strided = flare.flare_lse_combine(packed, packed[n:], lse_out=L2, shape=tuple(O_st.shape),
                                      part_stride=packed.numel() // R)
    assert torch.equal(dense, strided) and torch.equal(L1, L2)
    whole = flare.flare_encode(s_d, K_d, V_d)
    S64, K64, V64 = seeds.astype(np.float64), K.astype(np.float64), V.astype(np.float64)
    Lo = _per_head(w.B, w.H, lambda b, h: oracle.encode_shard(S64[h], K64[b, h], V64[b, h])[1])
    assert float(np.max(np.abs(to_host(L1) - Lo))) <= LSE_TOL["bf16"]
    # one bf16 rounding apart at most from the unsharded encode
    diff = (dense.float() - whole.float()).abs()
    assert float(diff.max()) <= 4 * 2.0 ** -9 * float(whole.float().abs().max())


def test_nccl_world_of_one():
    """flarepp_mix_cp over a real NCCL process group of one rank: the all-gather
    of one row leaves every value as it was, so Y equals flarepp_mix's bit for bit."""
    import torch
    import torch.distributed as dist

    require_cuda()
    w = inputs.custom(1, 4, 5000, 64, 32, dtype="bf16", seed_index=62)
    seeds, K, V = inputs.make_inputs(w)
    s_d, K_d, V_d = (to_dev(x, "bf16") for x in (seeds, K, V))
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        Y = cp.flarepp_mix_cp(s_d, K_d, V_d)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert flare.flare_check_status() == (0, 0)
    assert torch.equal(Y, flare.flarepp_mix(s_d, K_d, V_d))


def test_invalid_arguments():
    import torch

    require_cuda()
    O = torch.zeros((2, 1, 1, 16, 16), device="cuda")
    L = torch.zeros((2, 1, 1, 16), device="cuda")
    out = torch.empty((1, 1, 16, 16), device="cuda")
    lib = flare.lib()
    vp = __import__("ctypes").c_void_p
    for R, stride in ((0, 0), (2, -1)):
        rc = lib.flare_lse_combine(vp(O.data_ptr()), vp(L.data_ptr()), R, stride, vp(out.data_ptr()), None,
                                   1, 1, 16, 16, 0, None)
        assert rc == 1, (R, stride)
    K = torch.zeros((1, 1, 4, 16), device="cuda")
    rc = lib.flare_encode_lse(vp(out.data_ptr()), 0, vp(K.data_ptr()), vp(K.data_ptr()), vp(O.data_ptr()),
                              vp(L.data_ptr()), 1, 1, -1, 16, 16, 0, None, 0, None)
    assert rc == 1
    torch.cuda.synchronize()


# ---------------------------------------------------------------- sharded backward
def _emulate_save(s_d, K_d, V_d, R):
    """The sharded forward with save=True, R ranks emulated in turn: Q_dyn, Z
    and their log-sum-exps combined from all shards into one saved state."""
    import torch

    B, H, N, D = K_d.shape
    M = s_d.shape[-2]
    ops = cp.LibraryOps()
    saved = torch.empty(ops.saved_bytes(B, H, M, D, K_d.dtype), dtype=torch.uint8, device="cuda")
    Qv, Zv, L1, L2 = cp.saved_views(saved, B, H, M, D, K_d.dtype)
    recv = torch.empty((R, cp.exchange_floats(B, H, M, D)), dtype=torch.float32, device="cuda")
    shards = [(cp.shard_tokens(K_d, R, r), cp.shard_tokens(V_d, R, r)) for r in range(R)]
    for Q, out, lse in ((s_d, Qv, L1), (Qv, Zv, L2)):
        for r, (Kr, Vr) in enumerate(shards):
            ops.encode_lse(Q, Kr, Vr, recv[r])
        ops.combine(recv, B, H, M, D, K_d.dtype, out, lse)
    return saved, shards


def _emulate_backward(s_d, shards, dYs, saved, R):
    """The four phases on every emulated rank, with the sum over ranks of the
    exchange buffers (what the all-reduce returns) between phases."""
    import torch

    ops = cp.LibraryOps()
    B, H, _, D = shards[0][0].shape
    M = s_d.shape[-2]
    lat = B * H * M * D
    states = [ops.backward_state(s_d, Kr, M) for Kr, _ in shards]
    grads = [(torch.empty_like(s_d), torch.empty_like(Kr), torch.empty_like(Vr)) for Kr, Vr in shards]
    for phase, n in ((0, 2 * lat), (1, lat), (2, H * M * D), (3, 0)):
        for r in range(R):
            ops.backward_phase(phase, s_d, shards[r][0], shards[r][1], dYs[r], saved, states[r][0], states[r][1],
                               grads[r])
        if n:
            total = torch.stack([st[0][:n] for st in states]).sum(0)
            for st in states:
                st[0][:n].copy_(total)
    return grads


def test_sharded_backward_one_rank_matches_saved():
    """One rank, no exchange: the four phases give flarepp_mix_backward_saved's bits."""
    import torch

    require_cuda()
    w = inputs.custom(1, 2, 700, 256, 64, dtype="bf16", seed_index=90)
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    dev = [to_dev(x, "bf16") for x in (seeds, K, V, dY)]
    _, saved = flare.flarepp_mix_save(*dev[:3])
    want = flare.flarepp_mix_backward_saved(*dev, saved)
    got = _emulate_backward(dev[0], [(dev[1], dev[2])], [dev[3]], saved, 1)[0]
    for a, b in zip(got, want):
        assert torch.equal(a, b)
    assert flare.flare_check_status() == (0, 0)


@pytest.mark.parametrize("name,R", [("cloud", 3), ("long", 2), ("tiny_f32", 2)])
def test_sharded_backward_emulated_ranks(name, R):
    """R ranks: dK and dV of each rank's tokens and the common d_seeds, against
    the oracle's backward of the stored chain (the sharded forward's Q_dyn, Z)."""
    import torch

    require_cuda()
    w = inputs.WORKLOADS[name]
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    s_d, K_d, V_d, dY_d = (to_dev(x, w.dtype) for x in (seeds, K, V, dY))
    saved, shards = _emulate_save(s_d, K_d, V_d, R)
    dYs = [cp.shard_tokens(dY_d, R, r) for r in range(R)]
    grads = _emulate_backward(s_d, shards, dYs, saved, R)
    assert flare.flare_check_status() == (0, 0)
    for g in grads[1:]:
        assert torch.equal(g[0], grads[0][0])  # the same summed d_seeds on every rank
    got = [to_host(grads[0][0]), to_host(torch.cat([g[1] for g in grads], dim=2)),
           to_host(torch.cat([g[2] for g in grads], dim=2))]
    Qv, Zv, _, _ = cp.saved_views(saved, w.B, w.H, w.M, w.D, K_d.dtype)
    want = oracle.flarepp_backward(*(x.astype(np.float64) for x in (seeds, K, V, dY)), Q_dyn=to_host(Qv),
                                   Z=to_host(Zv))
    tensor_cores = w.dtype == "bf16" and w.D <= 64
    for label, g, r in zip(("d_seeds", "dK", "dV"), got, want):
        assert_backward_bar(f"{name}.cp{R}.{label}", g, r, w.dtype, tensor_cores)


def test_sharded_backward_with_an_empty_rank():
    """3 tokens over 5 ranks: the two ranks without tokens contribute zeros."""
    import torch

    require_cuda()
    w = inputs.custom(2, 2, 3, 16, 16, dtype="f32", seed_index=91)
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    s_d, K_d, V_d, dY_d = (to_dev(x, "f32") for x in (seeds, K, V, dY))
    saved, shards = _emulate_save(s_d, K_d, V_d, 5)
    grads = _emulate_backward(s_d, shards, [cp.shard_tokens(dY_d, 5, r) for r in range(5)], saved, 5)
    assert flare.flare_check_status() == (0, 0)
    want = oracle.flarepp_backward(*(x.astype(np.float64) for x in (seeds, K, V, dY)))
    got = [to_host(grads[0][0]), to_host(torch.cat([g[1] for g in grads], dim=2)),
           to_host(torch.cat([g[2] for g in grads], dim=2))]
    for g, r in zip(got, want):
        assert np.max(np.abs(g - r)) <= 1e-4


def test_nccl_world_of_one_training_step():
    """flarepp_mix_cp(save=True) and flarepp_mix_backward_cp over a real NCCL
    group of one rank: the same Y as flarepp_mix; gradients within the
    backward's bars of the single-GPU saved-state backward."""
    import torch
    import torch.distributed as dist

    require_cuda()
    w = inputs.custom(1, 2, 3000, 64, 32, dtype="bf16", seed_index=92)
    seeds, K, V = inputs.make_inputs(w)
    dY = inputs.make_upstream(w)
    s_d, K_d, V_d, dY_d = (to_dev(x, "bf16") for x in (seeds, K, V, dY))
    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        Y, saved = cp.flarepp_mix_cp(s_d, K_d, V_d, save=True)
        grads = cp.flarepp_mix_backward_cp(s_d, K_d, V_d, dY_d, saved)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert flare.flare_check_status() == (0, 0)
    assert torch.equal(Y, flare.flarepp_mix(s_d, K_d, V_d))
    Qv, Zv, _, _ = cp.saved_views(saved, 1, 2, 64, 32, torch.bfloat16)
    want = oracle.flarepp_backward(*(x.astype(np.float64) for x in (seeds, K, V, dY)), Q_dyn=to_host(Qv),
                                   Z=to_host(Zv))
    for label, g, r in zip(("d_seeds", "dK", "dV"), grads, want):
        assert_backward_bar(f"nccl1.{label}", to_host(g), r, "bf16", True)
