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
