"""GPU parity of the host-resident K/V tier (hga_forward mode
HGA_PREFILL_HOSTKV): K and V stay in pinned host RAM, only summaries and the
routed and fixed-window rows of each wave of query blocks reach the GPU.

The tier runs the same arithmetic as the in-HBM prefill (keys are rotated
with the same rounding when they are fetched), so its routed sets and
outputs must equal that path's bit for bit; outputs are also checked against
the CPU oracle on the routed sets.  Cases span several waves (32 blocks
each), a ragged last block, F = 0 / L = 0, MHA with D = 64, B > 1 and a warm
cache smaller than the sequence's groups; the bytes the tier reads over the
link are checked against bounds that follow from the routed sets.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, row_rel_err
from workloads import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu

SMALLLM = WORKLOADS["smalllm40m_bf16_prefill_4k"]
QWEN = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"]
HOST = WORKLOADS["qwen3_30b_a3b_bf16_hosttier_prefill_64k"]

CASES = {
    "qwen_3_waves_ragged": QWEN.replace(T=64 * 70 + 37),
    "qwen_one_wave": QWEN.replace(T=1024),
    "qwen_F0_L0": QWEN.replace(T=64 * 40, F=0, L=0, K_c=5, K_g=9),
    "smalllm_B2_D64": SMALLLM.replace(B=2, T=64 * 66),
    "qwen_L1_F3": QWEN.replace(T=64 * 33 + 5, F=3, L=1, K_c=4, K_g=7),
    # 800 groups per KV head against a warm cache of two waves' worth
    # (2 x 32 x 3 = 192 slots): slots are evicted and reused across 7 waves
    "qwen_cache_evicts": QWEN.replace(T=64 * 200, K_c=2, K_g=3),
}


def _hp(w):
    import hierarchical_kv_routing_b200 as hga
    return hga.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                         rope_theta=w.theta)


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def _run_pair(hga, w, seed):
    q, k, v, pos, _ = make_prefill_inputs(w, seed=seed)
    dev = torch.device("cuda")
    qd, pd = q.to(dev), pos.to(dev)
    hp = _hp(w)
    ref = hga.hga_forward_prefill(qd, k.to(dev), v.to(dev), pd, hp, want_lse=True,
                                  want_sel=True)
    kh, vh = k.pin_memory(), v.pin_memory()
    tier = hga.hga_forward_prefill_hostkv(qd, kh, vh, pd, hp, want_lse=True, want_sel=True)
    torch.cuda.synchronize()
    return (q, k, v, pos), ref, tier


@pytest.mark.parametrize("name", list(CASES))
def test_hosttier_equals_hbm_path_and_oracle(gpu_lib, name):
    w = CASES[name]
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=5)
    assert torch.equal(tier["sel_chunk"], ref["sel_chunk"])
    assert torch.equal(tier["sel_group"], ref["sel_group"])
    assert torch.equal(_bits(tier["out"]), _bits(ref["out"]))
    assert torch.equal(_bits(tier["lse"]), _bits(ref["lse"]))

    # oracle on sampled blocks of every wave over the routed sets
    T = pos.shape[1]
    NB = (T + 63) // 64
    blocks = sorted({0, 1, w.F + w.L + 1, 31, 32, 33, NB // 2, NB - 2, NB - 1} & set(range(NB)))
    units = [(b, u) for b in range(w.B) for u in blocks]
    sg = tier["sel_group"].cpu().numpy()
    force = np.stack([sg[b, u] for (b, u) in units])
    orc = oracle.hga(q, k, v, pos, oracle.Params.of(w), units=units, sel_g_force=force)
    O = tier["out"].float().cpu().numpy()
    for (b, u) in units:
        sl = slice(64 * u, min(T, 64 * u + 64))
        e = row_rel_err(O[b, sl], orc["O"][b, sl])
        assert e <= TOL[w.dtype], f"output rel err {e} at b={b} block={u}"


def test_hosttier_twice_in_a_row(gpu_lib):
    """Back-to-back calls reuse the side stream, events and staging buffers."""
    w = QWEN.replace(T=64 * 70)
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=9)
    hp = _hp(w)
    dev = torch.device("cuda")
    again = gpu_lib.hga_forward_prefill_hostkv(q.to(dev), k.pin_memory(), v.pin_memory(),
                                               pos.to(dev), hp)
    torch.cuda.synchronize()
    assert torch.equal(_bits(again["out"]), _bits(ref["out"]))


def test_hosttier_rejects_pageable_memory(gpu_lib):
    """Host arrays that are not pinned are refused by the binding; the C entry
    point checks again through the driver before launching anything."""
    import ctypes
    w = QWEN.replace(T=256)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=1)
    dev = torch.device("cuda")
    with pytest.raises(gpu_lib.HGAError):
        gpu_lib.hga_forward_prefill_hostkv(q.to(dev), k, v, pos.to(dev), _hp(w))
    lib = gpu_lib.load()
    hp = _hp(w).c()
    dims = gpu_lib._dims(w.B, w.T, w.Hq, w.Hkv, w.D, 1)
    io = gpu_lib._IO()
    qd, pd = q.to(dev), pos.to(dev)
    out = torch.empty_like(qd)
    io.q, io.k, io.v, io.pos, io.out = (qd.data_ptr(), k.data_ptr(), v.data_ptr(), pd.data_ptr(),
                                        out.data_ptr())
    n = int(lib.hga_workspace_size(2, ctypes.byref(dims), ctypes.byref(hp)))
    ws = torch.empty(n + 256, dtype=torch.uint8, device=dev)
    base = (ws.data_ptr() + 255) // 256 * 256
    st = lib.hga_forward(2, ctypes.byref(dims), ctypes.byref(hp), ctypes.byref(io),
                         ctypes.c_void_p(base), n, None)
    torch.cuda.synchronize()
    # HGA_ERR_INVALID_ARG; a driver that maps pageable memory for the GPU may
    # accept it, and then the result must still be right
    assert st in (0, 1)
    if st == 0:
        ref = gpu_lib.hga_forward_prefill(qd, k.to(dev), v.to(dev), pd, _hp(w))
        assert torch.equal(_bits(out), _bits(ref["out"]))


@pytest.mark.slow
def test_hosttier_64k_full_size(gpu_lib):
    """The 64K host-tier workload as the bench runs it: routed sets and
    outputs equal the in-HBM path's everywhere."""
    w = HOST
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=13)
    assert torch.equal(tier["sel_group"], ref["sel_group"])
    assert torch.equal(_bits(tier["out"]), _bits(ref["out"]))


def _fixed_link_bytes(w, T, W=32):
    """Bytes of sinks and windows the gathers read from host memory: the sink
    chunks for each of the first two waves, and each wave's window minus the
    tokens the previous wave's buffer already holds (same wave plan as the
    library: W-block waves, window from max(c0 - max(L, 1), F) to c1)."""
    C, NB, Lw = w.C, (T + w.C - 1) // w.C, max(w.L, 1)
    row = w.Hkv * w.D * 2 * 2                     # K and V of one token, all heads
    tokens, prev = 0, (0, 0)
    for wave, c0 in enumerate(range(0, NB, W)):
        c1 = min(c0 + W, NB)
        if wave < 2:
            tokens += min(w.F * C, T)
        nsink = min(c0, w.F)
        wlo = max(max(c0 - Lw, nsink), w.F)
        t0, t1 = wlo * C, max(min(c1 * C, T), wlo * C)
        held = max(0, min(t1, prev[1]) - max(t0, prev[0])) if wave > 0 else 0
        tokens += (t1 - t0) - held
        prev = (t0, t1)
    return w.B * tokens * row


def test_hosttier_warm_cache_link_bytes(gpu_lib):
    """The warm cache's traffic: every distinct routed group crosses the link
    at least once, and no group twice within a wave (at most the sum over
    waves of the wave's distinct groups); hits across waves make it less."""
    w = QWEN.replace(T=64 * 200, K_c=2, K_g=3)
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=11)
    assert torch.equal(_bits(tier["out"]), _bits(ref["out"]))
    dev = torch.device("cuda")
    gpu_lib.hga_hostkv_link_bytes(clear=True)
    gpu_lib.hga_forward_prefill_hostkv(q.to(dev), k.pin_memory(), v.pin_memory(), pos.to(dev),
                                       _hp(w))
    got = gpu_lib.hga_hostkv_link_bytes(clear=True)
    assert gpu_lib.hga_device_status(clear=True) == 0
    sg = tier["sel_group"].cpu().numpy()          # [B, NB, Hkv, K_g]
    group = w.g_s * w.D * 2 * 2                   # K and V rows of one group, one head
    lower = upper = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            ids = sg[b, :, h, :]
            lower += np.unique(ids[ids >= 0]).size
            for c0 in range(0, ids.shape[0], 32):
                wv = ids[c0:c0 + 32]
                upper += np.unique(wv[wv >= 0]).size
    routed = got - _fixed_link_bytes(w, w.T)
    assert lower * group <= routed <= upper * group, (lower, routed / group, upper)
    assert routed < upper * group          # some groups are served from the cache


def _clock_misses(sel_group, W, NS):
    """Misses of the warm tier's policy, replayed in plain Python: per wave the
    distinct routed groups, ascending; hits keep their slot; misses, ascending,
    take the first slots from the hand on that are free or were last used
    before the previous wave; the hand moves past the last slot taken."""
    B, NB, Hkv, _ = sel_group.shape
    misses = 0
    for b in range(B):
        for h in range(Hkv):
            slot_of, gid_of, stamp, hand = {}, [-1] * NS, [0] * NS, 0
            for wave, c0 in enumerate(range(0, NB, W)):
                ids = sel_group[b, c0:c0 + W, h, :].ravel()
                uniq = sorted(set(int(x) for x in ids if x >= 0))
                miss = []
                for g in uniq:
                    if g in slot_of:
                        stamp[slot_of[g]] = wave
                    else:
                        miss.append(g)
                victims = []
                for k in range(NS):
                    if len(victims) == len(miss):
                        break
                    s = (hand + k) % NS
                    if gid_of[s] < 0 or stamp[s] < wave - 1:
                        victims.append(s)
                assert len(victims) == len(miss)
                for s in victims:
                    if gid_of[s] >= 0:
                        del slot_of[gid_of[s]]
                for s, g in zip(victims, miss):
                    slot_of[g], gid_of[s], stamp[s] = s, g, wave
                if victims:
                    hand = (victims[-1] + 1) % NS
                misses += len(miss)
    return misses


def test_hosttier_warm_cache_follows_clock(gpu_lib):
    """The link bytes equal the sinks and windows plus exactly the misses the
    CLOCK policy has on these routed sets (a cache of 192 slots per KV head
    for 800 groups, so slots are evicted)."""
    w = QWEN.replace(T=64 * 200, K_c=2, K_g=3)
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=17)
    dev = torch.device("cuda")
    gpu_lib.hga_hostkv_link_bytes(clear=True)
    gpu_lib.hga_forward_prefill_hostkv(q.to(dev), k.pin_memory(), v.pin_memory(), pos.to(dev),
                                       _hp(w))
    got = gpu_lib.hga_hostkv_link_bytes(clear=True)
    ns = min((w.T // w.C) * (w.C // w.g_s), 2 * 32 * w.K_g)
    misses = _clock_misses(tier["sel_group"].cpu().numpy(), 32, ns)
    assert got == _fixed_link_bytes(w, w.T) + misses * w.g_s * w.D * 2 * 2


def test_hosttier_warm_cache_follows_the_workspace_budget(gpu_lib):
    """The warm tier sized by the caller's workspace (the pages' warm VRAM
    tier that shrinks to leave a headroom): from the smallest plan (one query
    block per wave, a two-wave cache of 2 K_g slots) through the default to
    the one that caches every group.  Every plan gives the in-HBM path's
    outputs bit for bit, and its link bytes are the sinks and windows of its
    wave size plus exactly the misses CLOCK has at its wave size and slot
    count."""
    w = QWEN.replace(T=64 * 200, K_c=2, K_g=3)
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=19)
    dev = torch.device("cuda")
    hp = _hp(w)
    sg = tier["sel_group"].cpu().numpy()
    bounds = gpu_lib.hga_hostkv_plan(w.B, w.T, w.Hq, w.Hkv, w.D, hp)
    default = gpu_lib.hga_workspace_size(gpu_lib.PREFILL_HOSTKV, w.B, w.T, w.Hq, w.Hkv, w.D,
                                         torch.bfloat16, hp)
    lo, hi = bounds["min_bytes"], bounds["max_bytes"]
    budgets = [lo, (lo + default) // 2, default, (default + hi) // 2, hi]
    plans = [gpu_lib.hga_hostkv_plan(w.B, w.T, w.Hq, w.Hkv, w.D, hp, nb) for nb in budgets]
    assert plans[0]["wave_blocks"] == 1 and plans[0]["cache_slots"] == 2 * w.K_g
    assert plans[2]["wave_blocks"] == 32 and plans[2]["cache_slots"] == 2 * 32 * w.K_g
    assert plans[-1]["cache_slots"] == (w.T // 64) * (64 // w.g_s)
    assert 1 < plans[1]["wave_blocks"] < 32 and plans[2]["cache_slots"] < plans[3]["cache_slots"]
    qd, kh, vh, pd = q.to(dev), k.pin_memory(), v.pin_memory(), pos.to(dev)
    group = w.g_s * w.D * 2 * 2
    for nb, plan in zip(budgets, plans):
        assert plan["bytes"] <= nb
        ws = torch.empty(nb, dtype=torch.uint8, device=dev)
        # the caching allocator hands out 512-byte aligned blocks, so all nb
        # bytes are usable
        assert ws.data_ptr() % 256 == 0
        gpu_lib.hga_hostkv_link_bytes(clear=True)
        res = gpu_lib.hga_forward_prefill_hostkv(qd, kh, vh, pd, hp, workspace=ws)
        got = gpu_lib.hga_hostkv_link_bytes(clear=True)
        assert gpu_lib.hga_device_status(clear=True) == 0
        assert res["plan"]["wave_blocks"] == plan["wave_blocks"]
        assert res["plan"]["cache_slots"] == plan["cache_slots"]
        assert torch.equal(_bits(res["out"]), _bits(ref["out"])), plan
        misses = _clock_misses(sg, plan["wave_blocks"], plan["cache_slots"])
        assert got == _fixed_link_bytes(w, w.T, plan["wave_blocks"]) + misses * group, plan
    # every group cached: each distinct routed (sequence, head, group) crosses once
    distinct = sum(np.unique(sg[b, :, h][sg[b, :, h] >= 0]).size
                   for b in range(w.B) for h in range(w.Hkv))
    assert _clock_misses(sg, 32, plans[-1]["cache_slots"]) == distinct


def test_hosttier_vram_headroom_sizes_the_cache(gpu_lib):
    """vram_headroom: the cache takes the device's free memory above the
    headroom, clamped to the plan's bounds; a headroom larger than the free
    memory gives the smallest plan, a zero headroom the largest."""
    w = QWEN.replace(T=64 * 200, K_c=2, K_g=3)
    hp = _hp(w)
    bounds = gpu_lib.hga_hostkv_plan(w.B, w.T, w.Hq, w.Hkv, w.D, hp)
    free, _ = torch.cuda.mem_get_info()
    small = gpu_lib.hostkv_workspace_bytes(w.B, w.T, w.Hq, w.Hkv, w.D, hp,
                                           vram_headroom=free + (1 << 30))
    big = gpu_lib.hostkv_workspace_bytes(w.B, w.T, w.Hq, w.Hkv, w.D, hp, vram_headroom=0)
    assert small == bounds["min_bytes"] and big == bounds["max_bytes"]


def test_hosttier_group_summaries_in_host_memory(gpu_lib):
    """Group summaries in the cold tier (the pages' store table keeps them in
    host RAM with the token K/V): stage 1 writes them into a pinned host table
    and routing reads the routed chunks' group rows over the link.  Routed
    sets and outputs are the in-HBM path's bit for bit, the host table holds
    exactly the summaries stage 1 builds on the GPU, and the link carries the
    table once plus, per block and KV head, the groups of its routed chunks."""
    w = QWEN.replace(T=64 * 70 + 37)
    (q, k, v, pos), ref, tier = _run_pair(gpu_lib, w, seed=23)
    dev = torch.device("cuda")
    hp = _hp(w)
    NC, gpc = w.T // 64, 64 // w.g_s
    sgh = torch.full((w.B, w.Hkv, NC * gpc, w.D), float("nan")).pin_memory()
    qd, kh, vh, pd = q.to(dev), k.pin_memory(), v.pin_memory(), pos.to(dev)
    gpu_lib.hga_hostkv_link_bytes(clear=True)
    gpu_lib.hga_forward_prefill_hostkv(qd, kh, vh, pd, hp)
    base = gpu_lib.hga_hostkv_link_bytes(clear=True)
    cold = gpu_lib.hga_forward_prefill_hostkv(qd, kh, vh, pd, hp, want_lse=True, want_sel=True,
                                              s_group_host=sgh)
    got = gpu_lib.hga_hostkv_link_bytes(clear=True)
    assert gpu_lib.hga_device_status(clear=True) == 0
    assert torch.equal(cold["sel_chunk"], ref["sel_chunk"])
    assert torch.equal(cold["sel_group"], ref["sel_group"])
    assert torch.equal(_bits(cold["out"]), _bits(ref["out"]))
    assert torch.equal(_bits(cold["lse"]), _bits(ref["lse"]))
    _, _, s_g = gpu_lib.hga_build_summaries(k.to(dev), pd, hp)
    torch.cuda.synchronize()
    assert torch.equal(sgh.view(torch.int32), s_g.cpu().view(torch.int32))
    NB = (w.T + 63) // 64
    rows = sum(min(w.K_c, max(0, c - w.L - 1 - w.F + 1)) for c in range(NB))
    assert got - base == (NC + rows) * gpc * w.D * 4 * w.B * w.Hkv
