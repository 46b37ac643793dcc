"""Host-side pieces of bench.py on CPU: the oracle baseline's job sampling (one
thread, a thread pool over (layer, sequence, kv head) units, sampled layers, the
append's encode timed on its own), on reduced workloads."""
import os

import bench
from workloads import WORKLOADS


def test_cpu_baseline_single_head_times_every_job():
    r = bench.cpu_baseline(WORKLOADS[1], 64, budget_s=0.2)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["unit"] == "GB/s"
    assert r["value"] > 0
    assert "every job of the step timed" in r["sample"]
    assert "threads" not in r          # one unit: nothing to spread over threads


def test_cpu_baseline_threads_and_append_encode():
    w = WORKLOADS[3].scaled(B=2, L=2048, append=64)
    r = bench.cpu_baseline(w, 64, budget_s=0.3, max_threads=2)
    assert r["value"] > 0 and r["append_encode_ms"] > 0
    if (os.cpu_count() or 1) >= 2:
        th = r["threads"]
        assert th["cores"] == 2 and th["value"] > 0 and th["nproc"] == os.cpu_count()


def test_cpu_baseline_samples_layers_and_scales():
    w = WORKLOADS[5].scaled(B=1, L=1024, layers=4)
    r = bench.cpu_baseline(w, 64, budget_s=0.2, max_threads=1)
    assert "layers [" in r["sample"] and "jobs (scaled)" in r["sample"]
    assert r["value"] > 0
