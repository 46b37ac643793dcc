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


def test_traffic_record_follows_the_decode_sources(tmp_path, monkeypatch):
    """The ncu traffic in the bench line is reported only while the decode kernel's
    sources (comments and white space aside) are the ones it was captured on."""
    import json
    import shutil
    csrc = tmp_path / "token_level_sparse_fwht_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.DECODE_SOURCES + ("encode.cu",):
        shutil.copy(os.path.join(bench.ROOT, "token_level_sparse_fwht_b200", "csrc", name),
                    csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.csrc_digest()
    rec = tmp_path / "traffic.json"
    rec.write_text(json.dumps({"cfg": {"csrc_sha": digest, "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(rec))
    assert bench.ncu_traffic("cfg") == 123
    assert bench.ncu_traffic("other") is None
    # an encoder edit or a comment in a decode source leaves the record valid ...
    (csrc / "encode.cu").write_text("// changed\n")
    with open(csrc / "decode.cu", "a") as f:
        f.write("\n// a comment\n")
    assert bench.csrc_digest() == digest and bench.ncu_traffic("cfg") == 123
    # ... a code change in one does not
    with open(csrc / "adamas_internal.cuh", "a") as f:
        f.write("\nnamespace extra_ns {}\n")
    assert bench.csrc_digest() != digest and bench.ncu_traffic("cfg") is None

