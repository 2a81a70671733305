"""Host-side pieces of bench.py: the low-rank plane width it gives a cache,
the algorithmic bytes its roofline divides by, and the kernel source hash that
ties committed traffic figures to the code they were measured on."""
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import get_workload  # noqa: E402


@pytest.mark.parametrize("d,dtype,D,want", [
    (32, "bf16", 128, 32), (16, "bf16", 128, 16), (64, "bf16", 128, 64), (12, "bf16", 128, 16),
    (128, "bf16", 128, 0), (121, "bf16", 128, 0), (16, "f32", 64, 16), (6, "f32", 64, 8), (64, "f32", 64, 0),
])
def test_lowrank_width(d, dtype, D, want):
    w = bench.lowrank_width(d, dtype, D)
    assert w == want
    if w:
        assert w >= d and (w * (2 if dtype == "bf16" else 4)) % 16 == 0 and w < D


def test_algorithmic_bytes_of_the_bench_workloads():
    # S*d*e low-rank key bytes plus k*2D*e gathered bytes per (batch, KV head) row
    for name, rows, S, d, k in [("llama2-7b-decode", 32, 4096, 32, 1024), ("llama3-8b-gqa-decode", 64, 32768, 64, 4096)]:
        w = get_workload(name)
        assert (w.rows, w.seq_len, w.d, w.k) == (rows, S, d, k)
        assert w.loki_bytes() == rows * (S * d * 2 + k * 2 * 128 * 2)
        assert w.dense_bytes() == rows * S * 2 * 128 * 2


def test_source_hash_ignores_comments_and_matches_committed_traffic():
    h = bench.source_hash()
    assert len(h) == 12
    assert bench._code_only("int a; // note\n/* block */ int b;") == bench._code_only("int a;\nint b;")
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        t = json.load(f)
    for workload, entry in t["loki_decode_step"].items():
        assert entry["dram_bytes_per_launch"] > get_workload(workload).loki_bytes()
        # the committed figures are used only while they describe the current code
        assert (bench.measured_traffic("loki_decode_step", workload) is not None) == (entry["source_hash"] == h)
