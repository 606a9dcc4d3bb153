"""Host logic of bench.py (CPU only): the roofline's bound by workload, the traffic record's gating by kernel
source, the visible-pair count against a closed form, the job throughput formula, prefix draws, and the clock
sampler's fallback when no GPU is visible."""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


PK = dict(hbm=6500.0, bf16=1600.0, bf16_sus=1400.0, src="measured")


def test_roofline_bound_follows_the_workload():
    r = bench.roofline("serving", tflops=400.0, gbs=3250.0, pk=PK, flops=1.0, nbytes=2.0)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == 6500.0 and abs(r["frac"] - 0.5) < 1e-12
    r = bench.roofline("qwen3_8b", tflops=400.0, gbs=3250.0, pk=PK, flops=1.0, nbytes=2.0)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and abs(r["frac"] - 0.25) < 1e-12


def test_traffic_is_reported_only_for_the_profiled_source(monkeypatch):
    h = hashlib.sha256()
    for rel in bench.ATTN_SOURCES:
        h.update(open(os.path.join(ROOT, rel), "rb").read())
    digest = h.hexdigest()
    monkeypatch.setattr(bench, "ATTN_TRAFFIC", {"qwen3_8b": {"bytes": 123.0, "source_sha256": digest},
                                                "serving": {"bytes": 456.0, "source_sha256": "0" * 64}})
    assert bench.attention_traffic("qwen3_8b") == 123.0
    assert bench.attention_traffic("serving") is None
    assert bench.attention_traffic("qwen3_30b_a3b") is None


def test_visible_pairs_closed_form():
    # a chain of N nodes under prefix P: node i sees P + i + 1 keys
    N, P = 9, 37
    parent = np.arange(-1, N - 1)[None]
    assert bench.visible_pairs(parent, [P]) == N * P + N * (N + 1) // 2
    # a star of N roots (parent -1 everywhere): each node sees P + 1
    assert bench.visible_pairs(-np.ones((1, N), np.int64), [P]) == N * (P + 1)


def test_ragged_visible_pairs_and_attention_work():
    # two sequences: a chain of 3 under P = 5, a star of 2 under P = 0
    parent = np.array([-1, 0, 1, -1, -1])
    offs, prefix = [0, 3, 5], [5, 0]
    pairs = bench.visible_pairs_ragged(parent, offs, prefix)
    assert pairs == (3 * 5 + 1 + 2 + 3) + (0 + 1 + 1)
    flops, nbytes = bench.attention_work([3, 2], 8, 2, prefix, pairs)
    assert flops == 4 * 128 * 8 * pairs
    kv = 2 * (5 + 3) * 128 * 4 + 2 * (0 + 2) * 128 * 4
    qo = 2 * 5 * 8 * 128 * 2
    meta = (4 * 1 + 4 * 3 + 12) + (4 * 1 + 4 * 2 + 12)
    assert nbytes == kv + qo + meta


def test_default_workload_is_the_largest_single_gpu_config():
    cfg = bench.WORKLOADS[bench.DEFAULT_WORKLOAD]
    size = lambda c: c["batch"] * c["budget"] * (c["prefix"] if isinstance(c["prefix"], int) else c["prefix"][1])
    assert all(size(cfg) >= size(c) for c in bench.WORKLOADS.values())


def test_job_throughput_counts_every_rank():
    assert bench.job_nodes_per_sec(2, 256, 4, 0.5) == 2 * 256 * 4 / 0.5e-3


def test_prefix_draws():
    rng = np.random.default_rng(0)
    cfg = dict(batch=50, prefix=(1024, 8192))
    p = bench.prefix_lengths(cfg, rng)
    assert len(p) == 50 and min(p) >= 1024 and max(p) <= 8192 and len(set(p)) > 1
    assert bench.prefix_lengths(dict(batch=3, prefix=4096), rng) == [4096] * 3


def test_clock_sampler_without_a_gpu(tmp_path):
    s = bench.NvmlSampler("GPU-00000000-0000-0000-0000-000000000000", str(tmp_path / "c.csv"))
    r = s.stop()
    assert "sm_mhz" in r and "reasons" in r
