"""The multi-rank path of the benchmark on CPU: two gloo ranks run the same
rank plumbing (rank_latent_attention_b200.ranks) that the GPU job runs over
NCCL, without a GPU.

Checked: each rank's cloud is its own batch element of the job's batch (the
inputs a single process generates for that batch element, bit for bit, and
different between ranks); the max over ranks reaches every rank; the job's
throughput counts all ranks' tokens over the slowest rank's time; only rank 0
reports.
"""
import hashlib
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from rank_latent_attention_b200 import inputs, ranks

BASE = inputs.custom(1, 2, 300, 32, 16, dtype="bf16", seed_index=41)


def _digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        env = ranks.RankEnv.from_environ()
        w = ranks.rank_workload(BASE, env.world)
        b = ranks.rank_batch_element(env)
        digests = [_digest(np.stack(inputs.make_head(w, b, h))) for h in range(w.H)]
        gathered = [None] * env.world
        dist.all_gather_object(gathered, {"rank": env.rank, "b": b, "digests": digests})
        slowest = ranks.max_over_ranks(10.0 + 3.0 * env.rank, env)
        value = ranks.job_tokens_per_s(w.N, env, slowest)
        rec = {"rank": env.rank, "world": env.world, "B": w.B, "gathered": gathered, "slowest": slowest,
               "value": value, "reports": ranks.reports(env)}
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump(rec, f)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a gloo rank did not finish")
        assert p.exitcode == 0
    recs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]

    # the job's batch: one cloud per rank
    job = ranks.rank_workload(BASE, world)
    assert all(r["B"] == world and r["world"] == world for r in recs)
    gathered = recs[0]["gathered"]
    assert [g["b"] for g in gathered] == [0, 1]
    for g in gathered:
        want = [_digest(np.stack(inputs.make_head(job, g["b"], h))) for h in range(job.H)]
        assert g["digests"] == want
    assert set(gathered[0]["digests"]).isdisjoint(gathered[1]["digests"])

    # slowest rank's time on every rank; whole-job tokens over it; rank 0 reports
    assert all(r["slowest"] == 13.0 for r in recs)
    assert all(r["value"] == pytest.approx(world * BASE.N / 13e-3) for r in recs)
    assert [r["reports"] for r in recs] == [True, False]
