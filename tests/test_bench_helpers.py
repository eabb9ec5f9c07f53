"""bench.py's host-side helpers: the committed ncu summary is read back as the traffic of
the update kernel only while the kernel source is the one it was taken on; the config
object and the byte counts the JSON line is built from."""
import os

import bench
import synthgen


def _recorded_hash():
    key = "kernels.cu sha256[:16]:"
    with open(os.path.join(bench.ROOT, "profiles", "adamw_cast_llama7b.md")) as f:
        return next(line[len(key):].strip() for line in f if line.startswith(key))


def test_profiled_traffic_follows_the_kernel_source(monkeypatch):
    # as if the kernel source were the one the summary was taken on
    monkeypatch.setattr(bench, "kernel_source_hash", _recorded_hash)
    t = bench.profiled_traffic("adamw_cast", "llama7b")
    assert isinstance(t, float) and 1.8e11 < t < 2.1e11  # ~29 B x 6.74e9 params
    # any other source: no traffic figure
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic("adamw_cast", "llama7b") is None
    assert bench.profiled_traffic("no_such_kernel", "llama7b") is None


def test_byte_counts():
    assert bench.schedule_bytes_per_param(8) == 50 and bench.model_bytes_per_param(8) == 42
    assert bench.schedule_bytes_per_param(1) == 36 and bench.model_bytes_per_param(1) == 28


def test_workload_config():
    wl = synthgen.workload("llama7b")
    c = bench.workload_config(wl, 14, wl.n, 1)
    assert c["workload"] == "llama7b_w8" and c["params"] == 6_738_415_616 and c["buckets"] == 14
    assert c["W"] == 8 and c["micro_batches"] == 1 and "337 GB" in c["l2"]
    c4 = bench.workload_config(wl, 14, wl.n, 8, micro=4)
    assert "replicas x8" in c4["parallelism"] and c4["micro_batches"] == 4
    assert "822 GB" in c4["l2"]  # (50 + 3 x 24) B per parameter
