"""The prefill benchmark's host arithmetic, on CPU.

* The algorithmic FLOP count equals a brute-force count over every chunk
  row, query head and visible key (4 * head_dim per key: q.k and p.v).
* A committed ncu summary feeds `traffic` only while every source it names
  still hashes to the recorded value.
* The oracle's CPU rate runs on a small batch and reports its sample.
"""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def test_prefill_flops_brute_force():
    b = workloads.prefill_custom("bf16", [5, 40, 1, 300], [5, 17, 1, 0], 8, 2, 64, 16, seed=2)
    want = 0
    for L, n in zip(b.context_lens, b.query_lens):
        for i in range(n):
            visible = L - n + i + 1
            want += b.num_q_heads * visible * 4 * b.head_dim
    assert bench.prefill_flops(b) == want


def test_profile_summary_gated_by_source_hash(tmp_path):
    src = os.path.join(ROOT, "paged_kv_cache_426_b200", "csrc", "pa_prefill.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    good = tmp_path / "good.md"
    good.write_text("# x\n\ntraffic_bytes_per_launch: 123\n"
                    f"source_sha256_16: pa_prefill.cu={h}\n")
    assert bench.profiled_fields(str(good))["traffic_bytes_per_launch"] == "123"
    stale = tmp_path / "stale.md"
    stale.write_text("traffic_bytes_per_launch: 123\nsource_sha256_16: pa_prefill.cu=0000000000000000\n")
    assert bench.profiled_fields(str(stale)) is None
    assert bench.profiled_fields(str(tmp_path / "missing.md")) is None


def test_prefill_cpu_baseline_small():
    b = workloads.prefill_custom("f16", [40, 90], [10, 90], 4, 2, 64, 16, seed=4)
    r = bench.prefill_cpu_baseline(b, 0.2)
    assert r["kind"] == "oracle" and r["unit"] == "TFLOP/s" and r["value"] > 0
    assert r["cores"] >= 1 and "chunk rows" in r["sample"]
