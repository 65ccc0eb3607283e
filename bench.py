"""Benchmark of the HGA routed-attention hot path on B200.

One step = the whole prefill path (mixed-RoPE summaries + K_rot, two-level
routing, tensor-core routed attention) over the Qwen3-30B-A3B-shaped 32K
workload (B=1, T=32768, 32 query / 4 KV heads, D=128, C=64, g_s=16, F=2,
L=8, K_c=16, K_g=32, planted-topic keys), seeded synthetic bf16 inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints one JSON line (rank 0).  With N > 1 (torchrun, one process per GPU)
every rank runs an independent replica of the workload (the path has no
cross-sequence exchange); value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import contextlib
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "qwen3_30b_a3b_bf16_prefill_32k"
METRIC = "HGA routed-attn prefill tokens/s & decode steps/s at 32K/64K; % HBM roofline"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attend_tc_qwen32k_traffic.txt")
CSRC = os.path.join(ROOT, "hierarchical_kv_routing_b200", "csrc")
ATTEND_SRC = os.path.join(CSRC, "attend_tc.cu")
DECODE_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_qwen64k_traffic.txt")
DECODE_SRC = os.path.join(CSRC, "decode.cu")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hga", choices=["hga", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-hosttier", action="store_true")
    ap.add_argument("--no-cold-l2", action="store_true")
    ap.add_argument("--no-smalllm", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--decode-replays", type=int, default=10)
    ap.add_argument("--decode-only", action="store_true",
                    help="profiling variant: only the decode part")
    ap.add_argument("--seq", type=int, default=0,
                    help="override the prefill length (small profiling cases only)")
    return ap.parse_args()


def max_over_ranks(x: float, device, world: int) -> float:
    """The largest of every rank's x (the job's time is its slowest rank's);
    every rank calls it at the same point."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Units per second of the whole job: every rank's units over the
    slowest rank's time."""
    return units_per_rank * world / (max_ms / 1e3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def params_of(w):
    import hierarchical_kv_routing_b200 as hga
    return hga.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                         rope_theta=w.theta)


def config_of(w, n):
    return {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D,
            "C": w.C, "g_s": w.g_s, "F": w.F, "L": w.L, "K_c": w.K_c, "K_g": w.K_g,
            "rope_theta": w.theta, "recipe": "planted-topic keys (sigma 0.5), queries at "
            "cosine 0.5 to one earlier middle chunk per block",
            "l2": "inputs larger than L2: Q and O stream 537 MB per step",
            "parallelism": "single GPU" if n == 1 else f"{n} independent replicas"}


def stage_bytes(w):
    """Compulsory HBM bytes of one summaries launch and one routing launch:
    every input read once and every output written once.  Summaries: K and
    positions in, rotated K and the chunk and group summary tables out.
    Routing: Q and positions in, the two summary tables read once, the chunk
    and group selections out, and for bf16 the rotated queries it hands to
    attention."""
    e = 2 if w.dtype == "bf16" else 4
    NC = w.T // w.C
    NB = (w.T + w.C - 1) // w.C
    tables = w.B * w.Hkv * NC * (1 + w.C // w.g_s) * w.D * 4
    kv = w.B * w.T * w.Hkv * w.D * e
    summaries = 2 * kv + w.B * w.T * 4 + tables
    route = (w.B * w.T * w.Hq * w.D * e + w.B * w.T * 4 + tables
             + w.B * NB * w.Hkv * (w.K_c + w.K_g) * 4)
    if w.dtype == "bf16":
        route += w.B * w.T * w.Hq * w.D * 2
    return summaries, route


def cold_l2_times(fns, stream, dev, iters=20):
    """Mean CUDA-event time of each call in fns with a cold L2: before every
    timed call a scratch buffer of twice the L2 size is written on the same
    stream, outside the events."""
    import torch
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 0) or 126 * 10**6)
    scratch = torch.empty(2 * l2 // 4 + 1024, dtype=torch.int32, device=dev)
    marks = []
    for it in range(iters + 2):                    # the first two are warm-up
        for n, fn in enumerate(fns):
            scratch.fill_(it)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            if it >= 2:
                marks.append((n, a, b))
    torch.cuda.synchronize(dev)
    out = [statistics.mean(a.elapsed_time(b) for m, a, b in marks if m == n)
           for n in range(len(fns))]
    del scratch
    return out


def cold_l2_report(cold, w, pk, src):
    """The line's cold_l2 entry: per stage its mean time, compulsory bytes,
    rate and fraction of the measured HBM copy peak; or the error text when
    the timing failed."""
    if not (isinstance(cold, list) and len(cold) == 2 and all(t > 0 for t in cold)):
        return {"error": str(cold)}
    hbm = pk.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    out = {"flush": "a scratch write of twice the L2 size before each timed call"}
    for name, t, nb in zip(("summaries", "route"), cold, stage_bytes(w)):
        out[name] = {"ms": t, "bytes": nb, "gbs": nb / t / 1e6, "frac": nb / t / 1e6 / hbm}
    out["peak_gbs"] = hbm
    out["peak_source"] = f"{src} hbm_gbs (copy)"
    return out


def attention_flops(w, sel_group):
    """Algorithmic FLOPs of one attention launch: for every query row,
    4 * D per visible key (2 for q.k, 2 for p.v), visible keys = fixed
    windows + routed groups + causal part of the own chunk."""
    import numpy as np
    sg = sel_group.cpu().numpy()                   # [B, NB, Hkv, K_g]
    B, NB = sg.shape[0], sg.shape[1]
    routed = (sg >= 0).sum(-1) * w.g_s             # [B, NB, Hkv]
    total = 0
    for c in range(NB):
        nsink = min(w.F, c)
        rec_lo = max(c - max(w.L, 1), nsink)
        fixed = (nsink + (c - rec_lo)) * w.C
        ncur = min(w.C, w.T - c * w.C)
        causal = ncur * (ncur + 1) // 2            # sum over tokens of (i - t0 + 1)
        keys_rows = (fixed + routed[:, c, :]) * ncur + causal   # [B, Hkv]
        total += int(keys_rows.sum()) * w.G
    return 4.0 * w.D * total


class ClockSampler:
    """Samples SM clock, max clock and active clock-event reasons via NVML on
    a background thread (reading only; nothing is changed), every `period`
    seconds.  `leg(name)` brackets a timed region so the result can give each
    region's own sample count and median clock."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index, period=0.0005):
        self.samples, self.max_mhz = [], None      # (time, MHz, reason bits)
        self.period = period
        self.legs = {}
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(device_index)
            bus = getattr(props, "pci_bus_id", None)
            dom = getattr(props, "pci_domain_id", 0)
            dev = getattr(props, "pci_device_id", 0)
            h = None
            if bus is not None:
                try:
                    h = pynvml.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{dev:02x}.0")
                except Exception:
                    h = None
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(0)
            self.h, self.nv = h, pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, r))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._ok:
            self.t.join()

    class _Leg:
        def __init__(self, owner, name):
            self.owner, self.name = owner, name

        def __enter__(self):
            self.t0 = time.perf_counter()

        def __exit__(self, *a):
            self.owner.legs.setdefault(self.name, []).append((self.t0, time.perf_counter()))

    def leg(self, name):
        return self._Leg(self, name)

    def _summary(self, samples):
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        reasons = set()
        for _, _, r in samples:
            for bit, name in self.REASONS.items():
                if r & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for _, m, _ in samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons - {"gpu_idle"}),
                "samples": len(samples)}

    def result(self):
        """Median clock and reasons over every bracketed leg (all samples when
        no leg was bracketed), plus each leg's own."""
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        spans = [sp for v in self.legs.values() for sp in v]
        inside = [x for x in self.samples if any(a <= x[0] <= b for a, b in spans)] \
            if spans else list(self.samples)
        out = self._summary(inside)
        out["period_ms"] = self.period * 1e3
        out["legs"] = {}
        for name, sp in self.legs.items():
            leg = self._summary([x for x in self.samples if any(a <= x[0] <= b for a, b in sp)])
            out["legs"][name] = {"samples": leg["samples"], "sm_mhz": leg["sm_mhz"],
                                 "reasons": leg["reasons"],
                                 "seconds": round(sum(b - a for a, b in sp), 4)}
        return out


def traffic_for_current_kernel(traffic_file=TRAFFIC_FILE, sources=(ATTEND_SRC,)):
    """Per-launch (or per-step) DRAM bytes from a committed ncu summary, only
    if that summary was taken on the current kernel source (the hash of the
    listed source files, in order, must match the one recorded)."""
    if not os.path.exists(traffic_file):
        return None
    h = hashlib.sha256()
    for f in sources:
        h.update(open(f, "rb").read())
    src_hash = h.hexdigest()[:16]
    vals = {}
    for line in open(traffic_file):
        if "=" in line and not line.startswith("#"):
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("source_sha256_16") != src_hash:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def _oracle_inputs(w, seed):
    import oracle
    from workloads import make_prefill_inputs
    q, k, v, pos, _ = make_prefill_inputs(w, seed=seed)
    return tuple(oracle._f64(x) for x in (q, k, v)) + (pos,)


def _oracle_sample(w, inputs, blocks, nthreads):
    import oracle
    q, k, v, pos = inputs
    t = time.perf_counter()
    oracle.hga(q, k, v, pos, oracle.Params.of(w), units=[(0, b) for b in blocks],
               nthreads=nthreads)
    return time.perf_counter() - t


def cpu_baseline(w, seed, budget_s=20.0, per_call=16):
    """The oracle (plain fp64 C; the full-sequence rotation and summary pass
    on one thread, then threads over (block, KV head) units) on a bounded
    sample of the workload, scaled to the whole workload's tokens/s."""
    inputs = _oracle_inputs(w, seed)
    nthreads = len(os.sched_getaffinity(0))
    t_pre = _oracle_sample(w, inputs, [], nthreads)
    NB = (w.T + w.C - 1) // w.C
    done, spent, t_blocks, i = 0, 0.0, 0.0, 0
    while spent < budget_s and done < NB:
        blocks = [(NB // 3 + (i * per_call + j) * 97) % NB for j in range(per_call)]
        i += 1
        dt = _oracle_sample(w, inputs, blocks, nthreads)
        spent += dt
        t_blocks += max(dt - t_pre, 0.0)
        done += len(blocks)
    est = t_pre + t_blocks / done * NB * w.B
    return {"value": w.B * w.T / est, "unit": "tokens/s",
            "cores": min(nthreads, per_call * w.Hkv), "kind": "oracle",
            "sample": f"{done} of {NB} query blocks (all {w.Hkv} KV heads each), {per_call} per "
                      f"call, after a {t_pre:.2f} s full-sequence pass; whole-workload time = that "
                      f"pass + mean block time x {NB}"}


def run_reference(args):
    """The CPU oracle on the same workload (rank 0 only).  Each step is a
    bounded sample: the full-sequence rotation and summary pass plus enough
    query blocks (all KV heads each) to give every host thread one (block,
    KV head) unit.  ms_per_step is the measured time of such a sampled step;
    value extrapolates it to the whole workload (that pass + mean block time
    x blocks)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from workloads import WORKLOADS
    w = WORKLOADS[WORKLOAD]
    inputs = _oracle_inputs(w, args.seed)
    nthreads = len(os.sched_getaffinity(0))
    per_step = max(1, -(-nthreads // w.Hkv))
    t_pre = _oracle_sample(w, inputs, [], nthreads)
    NB = w.T // w.C
    step_est, step_meas = [], []
    for s in range(args.warmup + args.steps):
        blocks = [(s * 97 * per_step + j * 211 + 11) % NB for j in range(per_step)]
        dt = _oracle_sample(w, inputs, blocks, nthreads)
        if s >= args.warmup:
            step_meas.append(dt)
            step_est.append(t_pre + max(dt - t_pre, 0.0) / per_step * NB)
    est = statistics.median(step_est)
    value = w.B * w.T / est
    cores = min(nthreads, per_step * w.Hkv)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.mean(step_meas) * 1e3,
            "ms_per_step_is": "the measured time of one sampled step (see cpu_baseline.sample); "
                              "value is the whole workload's tokens over the extrapolated "
                              "whole-workload time",
            "whole_workload_ms_estimate": est * 1e3,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle",
                             "sample": f"each step: {per_step} of {NB} query blocks (all "
                                       f"{w.Hkv} KV heads, one (block, KV head) unit per "
                                       f"thread on {cores} threads) after a {t_pre:.2f} s "
                                       f"full-sequence pass; whole-workload time = that pass "
                                       f"+ mean block time x {NB}; median over steps"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


DECODE_WORKLOAD = "qwen3_30b_a3b_bf16_decode_64k"


def decode_bytes_per_step(w, T0, steps):
    """Algorithmic HBM bytes of one decode step (average over the run): per
    (sequence, KV head) the middle-chunk summary rows scanned, the group rows
    of the routed chunks, the visible keys' K and V rows, and the step's own
    q / k / v / cache writes / output."""
    e = 2  # bf16
    total = 0
    for s in range(steps):
        t = T0 + s
        c = t // w.C
        n_mid = max(0, (c - w.L - 1 if w.L > 0 else c - 2) - w.F + 1)
        kc = min(w.K_c, n_mid)
        kg = min(w.K_g, kc * (w.C // w.g_s))
        nsink = min(w.F, c)
        rec_lo = max(c - max(w.L, 1), nsink)
        keys = (nsink + (c - rec_lo)) * w.C + kg * w.g_s + (t - c * w.C + 1)
        per_head = (n_mid * w.D * 4 + kc * (w.C // w.g_s) * w.D * 4 + keys * w.D * e * 2
                    + w.G * w.D * e * 2 + 2 * w.D * e + 3 * w.D * e)
        total += per_head * w.Hkv * w.B
    return total / steps


def bench_decode(args, dev, world, clk=None):
    """16 sequences with a 64K-token cache, 256 decode steps captured in one
    CUDA graph; steps/s and the HBM roofline of a step."""
    import torch
    import torch.distributed as dist

    import hierarchical_kv_routing_b200 as hga
    from workloads import WORKLOADS, make_decode_inputs
    w = WORKLOADS[DECODE_WORKLOAD]
    S = w.steps
    hp = params_of(w)
    d = make_decode_inputs(w, seed=args.seed + 1000 * (int(os.environ.get("RANK", "0")) + 1),
                           device=dev)
    cap = w.T + S
    cache = hga.KVCache(w.B, cap, w.Hkv, w.D, torch.bfloat16, hp, device=dev)
    hga.hga_fill_cache(d["k_hist"], d["v_hist"], d["pos_hist"], cache, hp)
    del d["k_hist"], d["v_hist"]
    ws = hga.decode_workspace(w.B, cap, w.Hq, w.Hkv, w.D, torch.bfloat16, hp, device=dev)
    outs = torch.empty(S, w.B, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
    q, kn, vn, pn = d["q"], d["k_new"], d["v_new"], d["pos_new"]

    def run_steps():
        for s in range(S):
            hga.hga_forward_decode(q[s], kn[s], vn[s], pn[s], cache, hp, out=outs[s],
                                   workspace=ws)

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        for _ in range(2):
            cache.lens.fill_(w.T)
            run_steps()
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    cache.lens.fill_(w.T)
    with torch.cuda.graph(graph):
        run_steps()
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        cache.lens.fill_(w.T)
        graph.replay()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    times = []
    for _ in range(args.decode_replays):
        cache.lens.fill_(w.T)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with (clk.leg("decode") if clk else contextlib.nullcontext()):
            e0.record(stream)
            graph.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
        times.append(e0.elapsed_time(e1))
    assert int(cache.lens[0].item()) == cap
    ms_step = max_over_ranks(sum(times), dev, world) / (len(times) * S)
    del graph
    pk, src = peaks()
    bps = decode_bytes_per_step(w, w.T, S)
    achieved = bps / (ms_step / 1e3) / 1e9
    return {"metric": "decode steps/s", "value": whole_job_rate(1, world, ms_step), "unit": "steps/s",
            "tokens_per_s": whole_job_rate(w.B, world, ms_step), "ms_per_step": ms_step,
            "steps_per_replay": S, "replays": len(times),
            "config": {"workload": w.name, "B": w.B, "cache_tokens": f"{w.T}..{cap - 1}",
                       "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "K_c": w.K_c, "K_g": w.K_g,
                       "graph": f"{S} steps captured in one CUDA graph, lens reset between "
                                "replays outside the timed events"},
            "gpu_launches_per_step": 3,   # scan, fixed-key and routed slices
            "roofline": {"bound": "hbm", "achieved": achieved,
                         "peak": pk.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]), "unit": "GB/s",
                         "frac": achieved / pk.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"]),
                         "traffic": traffic_for_current_kernel(DECODE_TRAFFIC_FILE,
                                                               (DECODE_SRC,)),
                         "bytes_per_step": bps,
                         "peak_source": f"{src} hbm_gbs (copy)"}}


HOSTTIER_WORKLOAD = "qwen3_30b_a3b_bf16_hosttier_prefill_64k"


def hosttier_link_bytes_uncached(w, sel_group):
    """Bytes over the host link for one host-tier prefill without the warm
    cache: raw K once (summaries), K and V of every token once (sinks and
    fixed windows; window chunks shared by consecutive waves move on the
    device), and K and V of every routed group of every (block, KV head)."""
    row = w.Hkv * w.D * 2
    routed = int((sel_group >= 0).sum().item()) * w.g_s * w.D * 2 * 2
    return w.B * w.T * row + 2 * w.B * w.T * row + routed


def bench_hosttier(args, dev, world, clk=None):
    """The 64K prefill with K/V in pinned host RAM; tokens/s and the fraction
    of the host-to-device copy bandwidth measured in the same run."""
    import torch
    import torch.distributed as dist

    import hierarchical_kv_routing_b200 as hga
    from workloads import WORKLOADS, make_prefill_inputs
    w = WORKLOADS[HOSTTIER_WORKLOAD]
    hp = params_of(w)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=args.seed + 77, device=dev)
    kh, vh = k.cpu().pin_memory(), v.cpu().pin_memory()
    del k, v
    stream = torch.cuda.current_stream(dev)
    n = hga.hga_workspace_size(hga.PREFILL_HOSTKV, w.B, w.T, w.Hq, w.Hkv, w.D, torch.bfloat16, hp)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    res = hga.hga_forward_prefill_hostkv(q, kh, vh, pos, hp, want_sel=True, workspace=ws)
    uncached = hosttier_link_bytes_uncached(w, res["sel_group"])
    for _ in range(max(2, min(args.warmup, 3))):
        hga.hga_forward_prefill_hostkv(q, kh, vh, pos, hp, out=out, workspace=ws)
    torch.cuda.synchronize(dev)
    hga.hga_hostkv_link_bytes(clear=True)
    if world > 1:
        dist.barrier()
    steps = 5
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (clk.leg("hosttier") if clk else contextlib.nullcontext()):
        e0.record(stream)
        for _ in range(steps):
            hga.hga_forward_prefill_hostkv(q, kh, vh, pos, hp, out=out, workspace=ws)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev, world)
    # bytes read over the link per call: the gathers' own count (sinks,
    # windows, warm-cache misses) plus stage 1's single pass over raw K
    link = hga.hga_hostkv_link_bytes(clear=True) / steps + w.B * w.T * w.Hkv * w.D * 2
    # host-to-device peak of this machine: copy engine, pinned source, 256 MiB
    src = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    best = 0.0
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dst.copy_(src, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize(dev)
        best = max(best, src.numel() / (a.elapsed_time(b) / 1e3) / 1e9)
    achieved = link / (ms / 1e3) / 1e9
    # the same prefill with the group summaries in the cold tier as well
    NC, gpc = w.T // w.C, w.C // w.g_s
    sgh = torch.empty(w.B, w.Hkv, NC * gpc, w.D, dtype=torch.float32).pin_memory()
    hga.hga_forward_prefill_hostkv(q, kh, vh, pos, hp, out=out, workspace=ws, s_group_host=sgh)
    torch.cuda.synchronize(dev)
    hga.hga_hostkv_link_bytes(clear=True)
    if world > 1:
        dist.barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with (clk.leg("hosttier") if clk else contextlib.nullcontext()):
        c0.record(stream)
        for _ in range(steps):
            hga.hga_forward_prefill_hostkv(q, kh, vh, pos, hp, out=out, workspace=ws,
                                           s_group_host=sgh)
        c1.record(stream)
        torch.cuda.synchronize(dev)
    ms_cold = max_over_ranks(c0.elapsed_time(c1) / steps, dev, world)
    link_cold = hga.hga_hostkv_link_bytes(clear=True) / steps + w.B * w.T * w.Hkv * w.D * 2
    return {"metric": "host-tier prefill tokens/s", "value": whole_job_rate(w.B * w.T, world, ms),
            "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "config": {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv,
                       "D": w.D, "K_c": w.K_c, "K_g": w.K_g,
                       "tier": "raw K and V in pinned host RAM; summaries, Q, O, two "
                               "32-block staging buffers and a warm cache of routed groups "
                               "in HBM"},
            "roofline": {"bound": "host link", "achieved": achieved, "peak": best,
                         "unit": "GB/s", "frac": achieved / best, "bytes_per_step": link,
                         "bytes_per_step_without_cache": uncached,
                         "peak_source": "measured in this run: pinned host -> device copy "
                                        "of 256 MiB, best of 5"},
            "group_summaries_in_host_memory": {
                "value": whole_job_rate(w.B * w.T, world, ms_cold), "unit": "tokens/s",
                "ms_per_step": ms_cold, "link_bytes_per_step": link_cold,
                "link_gbs": link_cold / (ms_cold / 1e3) / 1e9,
                "what": "the group summary table in pinned host RAM: written over the link by "
                        "stage 1, the routed chunks' group rows read over the link by routing"}}


def bench_backward(args, dev, world, clk, w, q, k_rot, v, pos, sel_g, hp, q_rot):
    """The backward of routed attention on the main workload (training
    through HGA attention): hga_attend_backward after one forward with LSE,
    given the rotated queries the forward's routing wrote, timed with CUDA
    events; the tensor-core roofline of its algorithmic work
    (five products per visible (row, key): S, dP, dQ, dK, dV, 2 D FLOPs each,
    i.e. 2.5 times the forward's; the recomputations of S and dP, for Delta
    and inside the dK/dV kernel, are not counted)."""
    import torch
    import torch.distributed as dist

    import hierarchical_kv_routing_b200 as hga
    stream = torch.cuda.current_stream(dev)
    out, lse = hga.hga_attend(q, pos, k_rot, v, sel_g, hp, want_lse=True)
    g = torch.Generator(device=dev).manual_seed(args.seed + 9)
    d_out = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(q.dtype)
    B, T, Hq, D = q.shape
    Hkv = k_rot.shape[2]
    f32 = dict(device=dev, dtype=torch.float32)
    dq = torch.empty(B, T, Hq, D, **f32)
    dk = torch.empty(B, T, Hkv, D, **f32)
    dv = torch.empty(B, T, Hkv, D, **f32)
    n = hga.hga_workspace_size(hga.ATTEND_BACKWARD, B, T, Hq, Hkv, D, q.dtype, hp)
    ws = torch.empty(n + 256, dtype=torch.uint8, device=dev)

    def call():
        hga.hga_attend_backward(q, pos, k_rot, v, sel_g, lse, d_out, hp, dq=dq, dk=dk, dv=dv,
                                workspace=ws, q_rot=q_rot)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize(dev)
    steps = max(5, min(args.steps, 20))
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clk.leg("backward"):
        e0.record(stream)
        for _ in range(steps):
            call()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev, world)
    flops = 2.5 * attention_flops(w, sel_g)
    pk, src = peaks()
    peak = pk.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    achieved = flops / (ms / 1e3) / 1e12
    return {"metric": "backward tokens/s", "value": whole_job_rate(w.B * w.T, world, ms),
            "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "config": {"workload": w.name, "what": "hga_attend_backward: dq, dk, dv (fp32) from "
                       "the forward's LSE and a random d_out; routed groups fixed"},
            "gpu_launches_per_step": 5,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak,
                         "flops_per_step": flops, "traffic": None,
                         "kernels": "k_bwd_prep, k_bwd_dq_tc, k_bwd_dkv_tc, k_bwd_finish "
                                    "(the call's whole time, all four kernels and two memsets)",
                         "peak_source": f"{src} bf16_tflops (burst)"}}


SMALLLM_WORKLOAD = "smalllm40m_bf16_prefill_4k"


def smalllm_bytes(w):
    """Compulsory HBM bytes of one prefill step of a workload: Q, K, V and O
    once each, and the rotated keys written once (the summary tables and the
    routed ids are under 2% more and are left out)."""
    e = 2 if w.dtype == "bf16" else 4
    return w.B * w.T * (2 * w.Hq + 3 * w.Hkv) * w.D * e


def bench_smalllm(args, dev, world, clk):
    """The SmallLM-40M-shaped prefill (8 sequences x 4096 tokens, 8 heads,
    D=64, MHA): the same three stages as the main step, timed with CUDA
    events; tokens/s and the HBM roofline of the step's compulsory bytes."""
    import torch
    import torch.distributed as dist

    import hierarchical_kv_routing_b200 as hga
    from workloads import WORKLOADS, make_prefill_inputs
    w = WORKLOADS[SMALLLM_WORKLOAD]
    hp = params_of(w)
    rank = int(os.environ.get("RANK", "0"))
    q, k, v, pos, _ = make_prefill_inputs(w, seed=args.seed + 500 + rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=args.seed + rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    k_rot, s_c, s_g = hga.hga_build_summaries(k, pos, hp)
    sel_c, sel_g = hga.hga_route(q, pos, s_c, s_g, hp)
    out = torch.empty_like(q)
    q_rot = torch.empty_like(q)             # routing hands the rotated queries to attention

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        hga.hga_build_summaries(k, pos, hp, k_rot=k_rot, s_chunk=s_c, s_group=s_g)
        if ev:
            ev[1].record(stream)
        hga.hga_route(q, pos, s_c, s_g, hp, sel_chunk=sel_c, sel_group=sel_g, q_rot=q_rot)
        if ev:
            ev[2].record(stream)
        hga.hga_attend(q, pos, k_rot, v, sel_g, hp, out=out, q_rot=q_rot)
        if ev:
            ev[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    flops = attention_flops(w, sel_g)
    steps = max(args.steps, 20)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    # the whole steps without stage events (they would serialise the
    # programmatic launches), then a second pass for the per-stage times
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clk.leg("smalllm"):
        t0.record(stream)
        for i in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    total_ms = max_over_ranks(t0.elapsed_time(t1), dev, world)
    for i in range(steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    stage_ms = [statistics.mean(e[a].elapsed_time(e[a + 1]) for e in evs) for a in range(3)]
    ms = total_ms / steps
    pk, src = peaks()
    hbm = pk.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    nb = smalllm_bytes(w)
    achieved = nb / (ms / 1e3) / 1e9
    tc = flops / (stage_ms[2] / 1e3) / 1e12
    tpk = pk.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    return {"metric": "prefill tokens/s", "value": whole_job_rate(w.B * w.T * steps, world, total_ms),
            "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
            "config": {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv,
                       "D": w.D, "F": w.F, "L": w.L, "K_c": w.K_c, "K_g": w.K_g,
                       "recipe": "chunk-topic keys (sigma 0.5); Q, V N(0,1)",
                       "l2": "Q, K, V, O and K_rot: 168 MB per step, above the 126 MB L2"},
            "stage_ms": {"summaries": stage_ms[0], "route": stage_ms[1], "attend": stage_ms[2]},
            "gpu_launches": 3 * steps,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "bytes_per_step": nb, "traffic": None,
                         "peak_source": f"{src} hbm_gbs (copy)",
                         "attention_tflops": tc, "attention_frac_of_bf16": tc / tpk,
                         "attention_flops_per_launch": flops}}


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import hierarchical_kv_routing_b200 as hga
    from workloads import WORKLOADS, make_prefill_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    hga.load()
    if args.decode_only:
        with ClockSampler(local) as clk:
            dec = bench_decode(args, dev, world, clk)
        dec["clocks"] = clk.result()
        if world > 1:
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"note": "profiling variant, not a bench line", "decode": dec}))
        return
    w = WORKLOADS[WORKLOAD]
    if args.seq:
        w = w.replace(T=args.seq, name=f"{w.name}_T{args.seq}")
    hp = params_of(w)

    q, k, v, pos, _ = make_prefill_inputs(w, seed=args.seed + rank, device=dev)
    stream = torch.cuda.current_stream(dev)
    k_rot, s_c, s_g = hga.hga_build_summaries(k, pos, hp)
    sel_c, sel_g = hga.hga_route(q, pos, s_c, s_g, hp)
    out = torch.empty_like(q)
    q_rot = torch.empty_like(q)             # routing hands the rotated queries to attention

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        hga.hga_build_summaries(k, pos, hp, k_rot=k_rot, s_chunk=s_c, s_group=s_g)
        if ev:
            ev[1].record(stream)
        hga.hga_route(q, pos, s_c, s_g, hp, sel_chunk=sel_c, sel_group=sel_g, q_rot=q_rot)
        if ev:
            ev[2].record(stream)
        hga.hga_attend(q, pos, k_rot, v, sel_g, hp, out=out, q_rot=q_rot)
        if ev:
            ev[3].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    flops = attention_flops(w, sel_g)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clk = ClockSampler(local).__enter__()     # runs until every leg is timed
    # The step's three launches run back to back (routing and attention are
    # programmatic dependents of the stage before them, so their set-up
    # overlaps it); events between the stages would serialise them, so the
    # per-stage times come from a second pass of the same steps.
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clk.leg("prefill"):
        t0.record(stream)
        for i in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    stage_ms = [statistics.mean(e[a].elapsed_time(e[a + 1]) for e in evs) for a in range(3)]
    total_ms = max_over_ranks(total_ms, dev, world)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(w.B * w.T * args.steps, world, total_ms)

    # summaries and routing again, each after a 2x-L2 scratch write (cold L2);
    # a failure here is reported in the line and never costs the bench line
    cold = None
    if not (args.no_cold_l2 or args.seq or args.no_e2e):   # full bench line only
        try:
            with clk.leg("cold_l2"):
                cold = cold_l2_times(
                    [lambda: hga.hga_build_summaries(k, pos, hp, k_rot=k_rot, s_chunk=s_c,
                                                     s_group=s_g),
                     lambda: hga.hga_route(q, pos, s_c, s_g, hp, sel_chunk=sel_c, sel_group=sel_g,
                                           q_rot=q_rot)],
                    stream, dev)
        except Exception as exc:               # noqa: BLE001 - reported, not raised
            cold = f"{type(exc).__name__}: {exc}"

    # end to end through the public one-call API, host buffers, every step's
    # copies inside the timed region; consecutive steps overlap as a serving
    # loop would run them: inputs in on one stream, the prefill on a second,
    # the output back on a third, over two sets of device buffers
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 20))
    hq, hk, hv, hpos = (x.cpu().pin_memory() for x in (q, k, v, pos))
    houts = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    ws = torch.empty(hga.hga_workspace_size(hga.PREFILL, w.B, w.T, w.Hq, w.Hkv, w.D,
                                            torch.bfloat16, hp) + 256,
                     dtype=torch.uint8, device=dev)
    dsets = [tuple(torch.empty(x.shape, dtype=x.dtype, device=dev) for x in (hq, hk, hv, hpos))
             for _ in range(2)]
    douts = [torch.empty(q.shape, dtype=q.dtype, device=dev) for _ in range(2)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for j in range(2):
        ev_comp[j].record(stream)
        ev_out[j].record(stream)

    def e2e_step(i):
        j = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[j])        # the prefill two steps back read set j
            for d, hsrc in zip(dsets[j], (hq, hk, hv, hpos)):
                d.copy_(hsrc, non_blocking=True)
            ev_in[j].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[j])
            s_comp.wait_event(ev_out[j])       # the read-out two steps back is done
            hga.hga_forward_prefill(*dsets[j], hp, out=douts[j], workspace=ws)
            ev_comp[j].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[j])
            houts[j].copy_(douts[j], non_blocking=True)
            ev_out[j].record(s_out)

    def join():
        for s_ in (s_in, s_comp, s_out):
            stream.wait_stream(s_)

    for i in range(2 if e2e_steps else 0):
        e2e_step(i)
    join()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with clk.leg("e2e"):
        e0.record(stream)
        for s_ in (s_in, s_comp, s_out):
            s_.wait_stream(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        join()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    te = max_over_ranks(e0.elapsed_time(e1), dev, world)
    e2e_value = whole_job_rate(w.B * w.T * e2e_steps, world, te) if e2e_steps else None
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hpos))
    d2h = houts[0].numel() * houts[0].element_size()

    bwd = None
    if not args.no_backward:
        try:
            bwd = bench_backward(args, dev, world, clk, w, q, k_rot, v, pos, sel_g, hp, q_rot)
        except Exception as exc:               # noqa: BLE001 - reported, not raised
            bwd = {"error": f"{type(exc).__name__}: {exc}"}
    dec = None if args.no_decode else bench_decode(args, dev, world, clk)
    tier = None if args.no_hosttier else bench_hosttier(args, dev, world, clk)
    small = None if (args.no_smalllm or args.seq) else bench_smalllm(args, dev, world, clk)
    clk.__exit__(None, None, None)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    pk, src = peaks()
    attend_s = stage_ms[2] / 1e3
    achieved = flops / attend_s / 1e12
    peak = pk.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic_for_current_kernel(),
            "kernel": "k_attend_tcp<128> (routed attention, tcgen05, persistent)",
            "flops_per_launch": flops, "avg_launch_ms": stage_ms[2],
            "peak_source": f"{src} bf16_tflops (burst; the kernel is timed alone per launch)"}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_of(w, world), "clocks": clk.result(),
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "api": "hga_forward(HGA_PREFILL) via the Python binding",
                    "overlap": "consecutive steps pipelined: inputs in, prefill and output "
                               "out on three streams over two device buffer sets"},
            "gpu_launches": 3 * args.steps,
            "stage_ms": {"summaries": stage_ms[0], "route": stage_ms[1], "attend": stage_ms[2]},
            "roofline": roof}
    if cold is not None:
        line["cold_l2"] = cold_l2_report(cold, w, pk, src)
    if dec is not None:
        line["decode"] = dec
    if tier is not None:
        line["hosttier"] = tier
    if small is not None:
        line["smalllm"] = small
    if bwd is not None:
        line["backward"] = bwd
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.seed)
    if args.seq or args.no_e2e:
        line["note"] = "profiling variant, not a bench line"
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
