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
    # (bf16: plus the rotated queries routing writes for attention)
    assert route == 2 * 32768 * 32 * 128 * 2 + 32768 * 4 + tables + 512 * 4 * (16 + 32) * 4
    assert 72e6 < summ < 73e6 and 542e6 < route < 543e6


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


def test_reference_arm_uses_every_host_thread_and_measures_its_step(monkeypatch, capsys):
    # one (block, KV head) unit per host thread, and ms_per_step is the time
    # the sampled step took, so steps x ms_per_step fits inside the run
    import argparse
    import json
    import time
    monkeypatch.setenv("RANK", "0")
    t0 = time.perf_counter()
    bench.run_reference(argparse.Namespace(gpus=1, steps=2, warmup=0, seed=0))
    wall_ms = (time.perf_counter() - t0) * 1e3
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    n = len(os.sched_getaffinity(0))
    w = WORKLOADS[bench.WORKLOAD]
    assert line["cpu_baseline"]["cores"] == min(n, -(-n // w.Hkv) * w.Hkv)
    assert line["steps"] * line["ms_per_step"] <= wall_ms
    assert line["whole_workload_ms_estimate"] >= line["ms_per_step"]


def test_smalllm_bytes():
    # Q and O (8 heads) and K, V, rotated K (8 KV heads): 168 MB at 8 x 4096
    w = WORKLOADS["smalllm40m_bf16_prefill_4k"]
    assert bench.smalllm_bytes(w) == 8 * 4096 * (2 * 8 + 3 * 8) * 64 * 2
    assert 167e6 < bench.smalllm_bytes(w) < 168e6


def test_clock_sampler_legs_without_nvml():
    # the per-leg summary counts only the samples inside each bracketed leg
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.max_mhz, s.period, s.legs, s._ok = [], 1965, 0.0005, {}, True
    s.samples = [(0.5, 1900, 0), (1.5, 1965, 0x4), (2.5, 1965, 0), (3.5, 1000, 0x1)]
    s.legs = {"prefill": [(1.0, 2.0)], "decode": [(2.0, 3.0)]}
    r = s.result()
    assert r["samples"] == 2 and r["sm_mhz"] == 1965 and r["reasons"] == ["sw_power_cap"]
    assert r["legs"]["prefill"]["samples"] == 1 and r["legs"]["decode"]["samples"] == 1
