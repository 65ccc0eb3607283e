"""Host-side arithmetic of bench.py, checked without a GPU."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import WORKLOADS  # noqa: E402


def test_stage_bytes_at_the_32k_workload():
    # summaries: K in and rotated K out (bf16), positions, chunk + 4 group
    # summaries per closed chunk and KV head (fp32); routing: Q, positions,
    # both tables once, K_c + K_g selected ids per block and KV head
    w = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"]
    summ, route = bench.stage_bytes(w)
    tables = 4 * 512 * (1 + 64 // 16) * 128 * 4
    assert summ == 2 * 32768 * 4 * 128 * 2 + 32768 * 4 + tables
    assert route == 32768 * 32 * 128 * 2 + 32768 * 4 + tables + 512 * 4 * (16 + 32) * 4
    assert 72e6 < summ < 73e6 and 274e6 < route < 275e6


def test_stage_bytes_count_a_ragged_tail_and_fp32():
    # an open last chunk has no summaries but its tokens are still moved
    w = WORKLOADS["tiny_f32_prefill_1k"].replace(T=1000)
    summ, route = bench.stage_bytes(w)
    NC, NB = 1000 // 64, (1000 + 63) // 64
    tables = w.B * w.Hkv * NC * (1 + 64 // w.g_s) * w.D * 4
    assert summ == 2 * 1000 * w.Hkv * w.D * 4 + 1000 * 4 + tables
    assert route == 1000 * w.Hq * w.D * 4 + 1000 * 4 + tables + NB * w.Hkv * (w.K_c + w.K_g) * 4


def test_cold_l2_report():
    w = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"]
    r = bench.cold_l2_report([0.05, 0.15], w, {"hbm_gbs": 6490.2}, "measured")
    summ, route = bench.stage_bytes(w)
    assert r["summaries"]["gbs"] == summ / 0.05 / 1e6          # bytes per ms -> GB/s
    assert abs(r["route"]["frac"] - route / 0.15 / 1e6 / 6490.2) < 1e-12
    assert r["peak_source"] == "measured hbm_gbs (copy)"
    # a failed timing is reported as text, never raised
    assert bench.cold_l2_report("RuntimeError: out of memory", w, {}, "fallback") == {
        "error": "RuntimeError: out of memory"}
    assert "error" in bench.cold_l2_report([0.0, 0.1], w, {}, "fallback")


def test_reference_arm_line_on_cpu(monkeypatch, capsys):
    # the reference arm is the oracle on host cores: one JSON line with the
    # same metric and workload as the library's line, its CPU baseline, and
    # an e2e entry that moves no bytes
    import argparse
    import json
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(argparse.Namespace(gpus=1, steps=1, warmup=0, seed=0))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True and line["value"] > 0
    assert line["config"]["workload"] == bench.WORKLOAD
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    e = line["e2e"]
    assert e["value"] == line["value"] and e["h2d_bytes_per_step"] == e["d2h_bytes_per_step"] == 0
