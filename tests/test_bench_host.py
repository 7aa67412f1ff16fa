"""Host-side helpers of bench.py (CPU): the oracle timings the bench line
reports next to the GPU numbers."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_blas_threads_reports_a_count_and_a_library():
    threads, api = bench.blas_threads()
    assert isinstance(threads, int) and threads >= 1
    assert isinstance(api, str) and api


def test_cpu_small_configs_times_every_small_workload():
    out = bench.cpu_small_configs()
    assert sorted(out) == ["c1", "c2", "c3", "c4"]
    for tag, r in out.items():
        assert r["workload"] == dict(bench.SMALL_CONFIGS)[tag]
        assert r["tokens_per_s"] > 0 and r["tokens_per_s_1_thread"] > 0
        assert r["head_ms"] > 0 and r["head_ms_1_thread"] > 0 and r["threads"] >= 1
