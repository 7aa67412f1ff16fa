"""The token-sharded mixer's plumbing (rank_latent_attention_b200.context_parallel)
on CPU: 2 and 3 gloo ranks run flarepp_mix_cp with the oracle's shard encode
and combine in place of the library's kernels, the collective being the same
torch.distributed all-gather.  The ranks' Y shards, put back in token order,
must equal the oracle's unsharded FLARE++ forward ("FLARE++" page,
"Contributions Clés", context-parallelism item: exact token sharding).
Includes ragged shards and a rank with no tokens.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from rank_latent_attention_b200 import context_parallel as cp


class OracleOps:
    """The four steps on CPU float64 tensors, through the oracle."""

    exchange_dtype = "float64"

    def __init__(self, group=None):
        self.group = group

    def encode_lse(self, Q, K, V, send):
        import oracle

        B, H, _, D = K.shape
        M = Q.shape[-2]
        O = np.zeros((B, H, M, D))
        L = np.zeros((B, H, M))
        for b in range(B):
            for h in range(H):
                q = (Q[b, h] if Q.dim() == 4 else Q[h]).numpy()
                O[b, h], L[b, h] = oracle.encode_shard(q, K[b, h].numpy(), V[b, h].numpy())
        n = O.size
        send[:n] = torch.from_numpy(O.reshape(-1))
        send[n:] = torch.from_numpy(L.reshape(-1))

    def all_gather(self, send):
        return cp.gather_rows(send, self.group)

    def combine(self, recv, B, H, M, D, dtype):
        import oracle

        n = B * H * M * D
        R = recv.shape[0]
        O = recv[:, :n].numpy().reshape(R, B, H, M, D)
        L = recv[:, n:].numpy().reshape(R, B, H, M)
        out = np.zeros((B, H, M, D))
        for b in range(B):
            for h in range(H):
                out[b, h] = oracle.combine_shards(list(O[:, b, h]), list(L[:, b, h]))[0]
        return torch.from_numpy(out)

    def decode(self, K, Q, Z):
        import oracle

        Y = np.zeros(K.shape)
        for b in range(K.shape[0]):
            for h in range(K.shape[1]):
                Y[b, h] = oracle.flare_decode(K[b, h].numpy(), Q[b, h].numpy(), Z[b, h].numpy())
        return torch.from_numpy(Y)


def _cloud(B, H, N, M, D, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal((H, M, D)) * 0.6, g.standard_normal((B, H, N, D)) * 0.6,
            g.standard_normal((B, H, N, D)) * 0.6)


def _rank_main(rank, world, port, out_dir, sizes):
    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        B, H, N, M, D, seed = sizes
        seeds, K, V = (torch.from_numpy(x) for x in _cloud(B, H, N, M, D, seed))
        Kr, Vr = cp.shard_tokens(K, world, rank), cp.shard_tokens(V, world, rank)
        send_floats = cp.exchange_floats(B, H, M, D)
        Y, Qd, Z = cp.flarepp_mix_cp(seeds, Kr, Vr, ops=OracleOps(), return_intermediates=True)
        np.save(os.path.join(out_dir, f"Y{rank}.npy"), Y.numpy())
        np.save(os.path.join(out_dir, f"Q{rank}.npy"), Qd.numpy())
        np.save(os.path.join(out_dir, f"Z{rank}.npy"), Z.numpy())
        with open(os.path.join(out_dir, f"meta{rank}.json"), "w") as f:
            json.dump({"range": cp.token_range(N, world, rank), "send": send_floats}, f)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,sizes", [
    (2, (2, 2, 37, 4, 3, 11)),   # ragged: 18 + 19 tokens
    (3, (1, 2, 2, 3, 2, 12)),    # 2 tokens over 3 ranks: rank 0 holds none
])
def test_sharded_mix_matches_oracle(tmp_path, world, sizes):
    import oracle

    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path), sizes)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0

    B, H, N, M, D, seed = sizes
    seeds, K, V = _cloud(B, H, N, M, D, seed)
    Qo, Zo, Yo = oracle.flarepp_mix(seeds, K, V)
    metas = [json.load(open(tmp_path / f"meta{r}.json")) for r in range(world)]
    assert [m["range"] for m in metas] == [list(cp.token_range(N, world, r)) for r in range(world)]
    assert metas[0]["range"][0] == 0 and metas[-1]["range"][1] == N
    Y = np.concatenate([np.load(tmp_path / f"Y{r}.npy") for r in range(world)], axis=2)
    assert Y.shape == Yo.shape
    assert np.allclose(Y, Yo, rtol=1e-12, atol=1e-13)
    for r in range(world):  # Q_dyn and Z are replicated, identical on every rank
        assert np.allclose(np.load(tmp_path / f"Q{r}.npy"), Qo, rtol=1e-12, atol=1e-13)
        assert np.allclose(np.load(tmp_path / f"Z{r}.npy"), Zo, rtol=1e-12, atol=1e-13)
        assert metas[r]["send"] == B * H * M * (D + 1)


def test_token_range_partitions():
    for N in (0, 1, 2, 7, 100, 1 << 20):
        for world in (1, 2, 3, 8):
            ranges = [cp.token_range(N, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == N
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0
    with pytest.raises(ValueError):
        cp.token_range(5, 2, 2)


class OracleTrainOps(OracleOps):
    """OracleOps plus the saved state and the four backward phases, in float64
    through the oracle's attention weights; the phases split the chain rule the
    way the library's kernels do (token-local terms, then sums over ranks)."""

    lse_dtype = torch.float64

    def saved_bytes(self, B, H, M, D, dtype):
        r = lambda x: (x + 255) // 256 * 256  # noqa: E731
        return 2 * r(B * H * M * D * 8) + 2 * r(B * H * M * 8)

    def combine(self, recv, B, H, M, D, dtype, out=None, lse_out=None):
        import oracle

        n = B * H * M * D
        R = recv.shape[0]
        O = recv[:, :n].numpy().reshape(R, B, H, M, D)
        L = recv[:, n:].numpy().reshape(R, B, H, M)
        res = np.zeros((B, H, M, D))
        lse = np.zeros((B, H, M))
        for b in range(B):
            for h in range(H):
                res[b, h], lse[b, h] = oracle.combine_shards(list(O[:, b, h]), list(L[:, b, h]))
        res = torch.from_numpy(res)
        if out is not None:
            out.copy_(res)
            lse_out.copy_(torch.from_numpy(lse))
        return res

    def all_reduce(self, t):
        return cp.all_reduce_sum(t, self.group)

    def backward_state(self, seeds, K, M):
        B, H, _, D = K.shape
        return torch.zeros(2 * B * H * M * D, dtype=torch.float64), {}

    def backward_phase(self, phase, seeds, K, V, dY, saved, exch, ws, grads):
        import oracle
        from oracle import flare_oracle

        B, H, N, D = K.shape
        M = seeds.shape[-2]
        Qd, Z, L1, L2 = (x.numpy() for x in cp.saved_views(saved, B, H, M, D, torch.float64, torch.float64))
        S = seeds.numpy()
        k, v, dy = K.numpy(), V.numpy(), dY.numpy()
        lat = B * H * M * D
        if phase == 0:
            ws["dK"], ws["dV"] = np.zeros((B, H, N, D)), np.zeros((B, H, N, D))
            dZ, dQd = np.zeros((B, H, M, D)), np.zeros((B, H, M, D))
            for b in range(B):
                for h in range(H):
                    P3 = oracle.attention_weights(k[b, h], Qd[b, h])  # local tokens x all latents
                    Y = P3 @ Z[b, h]
                    dS3 = flare_oracle._softmax_backward(P3, dy[b, h] @ Z[b, h].T, np.sum(dy[b, h] * Y, axis=1))
                    dZ[b, h] = P3.T @ dy[b, h]
                    dQd[b, h] = dS3.T @ k[b, h]
                    ws["dK"][b, h] = dS3 @ Qd[b, h]
            exch[:lat] = torch.from_numpy(dZ.reshape(-1))
            exch[lat:2 * lat] = torch.from_numpy(dQd.reshape(-1))
        elif phase == 1:
            ws["dZ"] = exch[:lat].numpy().reshape(B, H, M, D).copy()
            ws["dQd"] = exch[lat:2 * lat].numpy().reshape(B, H, M, D).copy()
            part = np.zeros((B, H, M, D))
            for b in range(B):
                for h in range(H):
                    A2 = np.exp(Qd[b, h] @ k[b, h].T - L2[b, h][:, None])  # global normalisation
                    dZ = ws["dZ"][b, h]
                    dS2 = flare_oracle._softmax_backward(A2, dZ @ v[b, h].T, np.sum(dZ * Z[b, h], axis=1))
                    part[b, h] = dS2 @ k[b, h]
                    ws["dV"][b, h] = A2.T @ dZ
                    ws["dK"][b, h] += dS2.T @ Qd[b, h]
            exch[:lat] = torch.from_numpy(part.reshape(-1))
        elif phase == 2:
            ws["dQd"] += exch[:lat].numpy().reshape(B, H, M, D)
            ds = np.zeros((H, M, D))
            for b in range(B):
                for h in range(H):
                    A1 = np.exp(S[h] @ k[b, h].T - L1[b, h][:, None])
                    dQ = ws["dQd"][b, h]
                    dS1 = flare_oracle._softmax_backward(A1, dQ @ v[b, h].T, np.sum(dQ * Qd[b, h], axis=1))
                    ds[h] += dS1 @ k[b, h]
                    ws["dV"][b, h] += A1.T @ dQ
                    ws["dK"][b, h] += dS1.T @ S[h]
            exch[:H * M * D] = torch.from_numpy(ds.reshape(-1))
        else:
            grads[0].copy_(exch[:H * M * D].reshape(H, M, D))
            grads[1].copy_(torch.from_numpy(ws["dK"]))
            grads[2].copy_(torch.from_numpy(ws["dV"]))


def _train_main(rank, world, port, out_dir, sizes):
    import torch.distributed as dist

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        B, H, N, M, D, seed = sizes
        seeds, K, V = (torch.from_numpy(x) for x in _cloud(B, H, N, M, D, seed))
        dY = torch.from_numpy(np.random.default_rng(seed + 1).standard_normal((B, H, N, D)))
        Kr, Vr, dYr = (cp.shard_tokens(x, world, rank) for x in (K, V, dY))
        ops = OracleTrainOps()
        Y, saved = cp.flarepp_mix_cp(seeds, Kr, Vr, ops=ops, save=True)
        ds, dK, dV = cp.flarepp_mix_backward_cp(seeds, Kr, Vr, dYr, saved, ops=ops)
        for name, x in (("Y", Y), ("ds", ds), ("dK", dK), ("dV", dV)):
            np.save(os.path.join(out_dir, f"{name}{rank}.npy"), x.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,sizes", [(2, (2, 2, 29, 3, 2, 21)), (3, (1, 2, 2, 4, 3, 22))])
def test_sharded_training_step_matches_oracle(tmp_path, world, sizes):
    """Forward with saved state and the four-phase backward on gloo ranks: Y,
    dK and dV of every rank's tokens and the summed d_seeds equal the oracle's
    unsharded forward and backward (the second case has a rank without tokens)."""
    import oracle

    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_train_main, args=(r, world, port, str(tmp_path), sizes)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0
    B, H, N, M, D, seed = sizes
    seeds, K, V = _cloud(B, H, N, M, D, seed)
    dY = np.random.default_rng(seed + 1).standard_normal((B, H, N, D))
    _, _, Yo = oracle.flarepp_mix(seeds, K, V)
    dso, dKo, dVo = oracle.flarepp_backward(seeds, K, V, dY)
    cat = lambda n: np.concatenate([np.load(tmp_path / f"{n}{r}.npy") for r in range(world)], axis=2)  # noqa: E731
    assert np.allclose(cat("Y"), Yo, rtol=1e-12, atol=1e-13)
    assert np.allclose(cat("dK"), dKo, rtol=1e-11, atol=1e-12)
    assert np.allclose(cat("dV"), dVo, rtol=1e-11, atol=1e-12)
    for r in range(world):  # every rank holds the same, summed, seed gradient
        assert np.allclose(np.load(tmp_path / f"ds{r}.npy"), dso, rtol=1e-11, atol=1e-12)
