"""GPU parity of the decode step against the oracle's full recompute.

A prompt fills the cache through hga_forward(HGA_PREFILL); then every decode
step appends one token per sequence, builds the summaries of a chunk when the
token closes it, routes with the token's own query and attends.  Each step's
output, LSE and routed sets are compared with the oracle run on the whole
sequence with per-token routing (the pages' "decode vs full recompute" check,
Table 7); the incrementally built summaries are compared with the oracle's
summaries of the final cache.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, RouteRef, check_unit_selection, row_rel_err
from workloads import WORKLOADS, make_decode_inputs

pytestmark = pytest.mark.gpu

QWEN = WORKLOADS["qwen3_30b_a3b_bf16_decode_64k"]
TINY = WORKLOADS["tiny_f32_prefill_1k"]

CASES = {
    # history, steps, capacity: every case crosses a chunk boundary
    "bf16_qwen_like": (QWEN.replace(B=2, Hq=8, Hkv=2), 640, 72, 768),
    "bf16_qwen_heads": (QWEN.replace(B=2), 700, 60, 832),
    "f32_ragged_prompt": (TINY.replace(B=2, Hq=4, Hkv=2), 200, 60, 320),
    "f32_L0_F0": (TINY.replace(B=1, F=0, L=0, K_c=3, K_g=5), 300, 40, 384),
    "bf16_D64_mha": (WORKLOADS["smalllm40m_bf16_prefill_4k"].replace(B=2, Hq=4, Hkv=4), 500, 30, 576),
}


def _hp(hga, w):
    return hga.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                         rope_theta=w.theta)


def _np(t):
    return t.detach().float().cpu().numpy()


def run_decode(hga, w, T_hist, steps, cap, seed, pos_mod=None):
    d = make_decode_inputs(w, seed=seed, T=T_hist, steps=steps)
    if pos_mod:
        d["pos_hist"] = (d["pos_hist"] % pos_mod).contiguous()
        d["pos_new"] = (d["pos_new"] % pos_mod).contiguous()
    dev = torch.device("cuda")
    dt = d["k_hist"].dtype
    hp = _hp(hga, w)
    cache = hga.KVCache(w.B, cap, w.Hkv, w.D, dt, hp, device=dev)
    q_hist = torch.randn(w.B, T_hist, w.Hq, w.D, generator=torch.Generator().manual_seed(seed)).to(dt)
    hga.hga_forward_prefill(q_hist.to(dev), d["k_hist"].to(dev), d["v_hist"].to(dev),
                            d["pos_hist"].to(dev), hp, cache=cache)
    ws = hga.decode_workspace(w.B, cap, w.Hq, w.Hkv, w.D, dt, hp, device=dev)
    outs, lses, selc, selg = [], [], [], []
    for s in range(steps):
        r = hga.hga_forward_decode(d["q"][s].to(dev), d["k_new"][s].to(dev), d["v_new"][s].to(dev),
                                   d["pos_new"][s].to(dev), cache, hp, want_lse=True,
                                   want_sel=True, workspace=ws)
        outs.append(r["out"])
        lses.append(r["lse"])
        selc.append(r["sel_chunk"])
        selg.append(r["sel_group"])
    torch.cuda.synchronize()
    return d, cache, torch.stack(outs), torch.stack(lses), torch.stack(selc), torch.stack(selg)


def check_decode(hga, case, seed=5, pos_mod=None):
    w, T_hist, steps, cap = case
    d, cache, out, lse, selc, selg = run_decode(hga, w, T_hist, steps, cap, seed=seed,
                                                pos_mod=pos_mod)
    Ttot = T_hist + steps
    K = torch.cat([d["k_hist"], d["k_new"].transpose(0, 1)], 1)
    V = torch.cat([d["v_hist"], d["v_new"].transpose(0, 1)], 1)
    pos = torch.cat([d["pos_hist"], d["pos_new"].transpose(0, 1)], 1)
    Q = torch.zeros(w.B, Ttot, w.Hq, w.D, dtype=torch.float64)
    Q[:, T_hist:] = d["q"].transpose(0, 1).double()
    p = oracle.Params.of(w)
    units = [(b, T_hist + s) for b in range(w.B) for s in range(steps)]
    sc, sg = selc.cpu().numpy(), selg.cpu().numpy()          # [S, B, Hkv, K]
    rr = oracle.hga(Q, K, V, pos, p, route_block=1, units=units, attend=False)
    ref = RouteRef(Q, K, pos, p, w.Hkv)
    for i, (b, t) in enumerate(units):
        s = t - T_hist
        for h in range(w.Hkv):
            ok, _ = check_unit_selection(ref, b, h, t, t + 1, t // 64, sc[s, b, h], sg[s, b, h],
                                         rr["sel_c"][i, h], rr["sel_g"][i, h])
            assert ok, f"routing mismatch b={b} t={t} h={h}"
    force = np.stack([sg[t - T_hist, b] for (b, t) in units])
    orc = oracle.hga(Q, K, V, pos, p, route_block=1, units=units, sel_g_force=force)
    O, L = _np(out), _np(lse)
    tol = TOL[w.dtype]
    for (b, t) in units:
        s = t - T_hist
        e = row_rel_err(O[s, b], orc["O"][b, t])
        assert e <= tol, f"decode output rel err {e} at b={b} t={t}"
        le = np.abs(L[s, b] - orc["LSE"][b, :, t]).max()
        assert le <= tol * max(1.0, np.abs(orc["LSE"][b, :, t]).max())
    # the cache: lens, positions, rotated keys, and incrementally built summaries
    assert (cache.lens.cpu() == Ttot).all()
    assert torch.equal(cache.pos[:, :Ttot].cpu(), pos)
    S_c, S_g = oracle.build_summaries(K, pos, p)
    nc = Ttot // 64
    assert row_rel_err(_np(cache.s_chunk[:, :, :nc]), S_c[:, :, :nc]) < 2e-6
    assert row_rel_err(_np(cache.s_group[:, :, :nc * (64 // w.g_s)]),
                       S_g[:, :, :nc * (64 // w.g_s)]) < 2e-6


@pytest.mark.parametrize("name", list(CASES))
def test_decode_parity(gpu_lib, name):
    check_decode(gpu_lib, CASES[name])


def test_decode_wrapped_positions(gpu_lib):
    """Positions modulo a period shorter than the sequence (the pages'
    position-mod-65536 variant at a small period): the steps cross a wrap
    and a chunk boundary; rotation uses the given positions, causality the
    token index."""
    check_decode(gpu_lib, CASES["bf16_qwen_like"], seed=8, pos_mod=677)


def test_decode_full_budget_is_dense(gpu_lib):
    w = TINY.replace(B=1, Hq=4, Hkv=2, K_c=64, K_g=256)
    d, cache, out, lse, _, _ = run_decode(gpu_lib, w, 300, 30, 384, seed=9)
    Ttot = 330
    K = torch.cat([d["k_hist"], d["k_new"].transpose(0, 1)], 1)
    V = torch.cat([d["v_hist"], d["v_new"].transpose(0, 1)], 1)
    pos = torch.cat([d["pos_hist"], d["pos_new"].transpose(0, 1)], 1)
    Q = torch.zeros(1, Ttot, w.Hq, w.D, dtype=torch.float64)
    Q[:, 300:] = d["q"].transpose(0, 1).double()
    O, _ = oracle.dense(Q, K, V, pos, w.theta)
    assert row_rel_err(_np(out)[:, 0], O[0, 300:]) <= 1e-5


@pytest.mark.slow
def test_decode_64k_full_size_graph(gpu_lib):
    """The bench's decode configuration: 16 sequences with a 65536-token cache,
    256 steps captured in one CUDA graph.  Every step's routed sets of two
    sampled sequences and sampled steps' outputs are checked against the
    oracle's full recompute; lens and the summaries of the chunks closed by
    the run are checked for all sequences."""
    hga = gpu_lib
    w = QWEN
    S = w.steps
    dev = torch.device("cuda")
    hp = _hp(hga, w)
    d = make_decode_inputs(w, seed=21, device=dev)
    cap = w.T + S
    cache = hga.KVCache(w.B, cap, w.Hkv, w.D, torch.bfloat16, hp, device=dev)
    hga.hga_fill_cache(d["k_hist"], d["v_hist"], d["pos_hist"], cache, hp)
    ws = hga.decode_workspace(w.B, cap, w.Hq, w.Hkv, w.D, torch.bfloat16, hp, device=dev)
    outs = torch.empty(S, w.B, w.Hq, w.D, dtype=torch.bfloat16, device=dev)
    sels = torch.empty(S, w.B, w.Hkv, w.K_g, dtype=torch.int32, device=dev)
    selc = torch.empty(S, w.B, w.Hkv, w.K_c, dtype=torch.int32, device=dev)
    import ctypes

    def run_steps():
        for s in range(S):
            io = hga._IO()
            io.q_new, io.k_new = d["q"][s].data_ptr(), d["k_new"][s].data_ptr()
            io.v_new, io.pos_new = d["v_new"][s].data_ptr(), d["pos_new"][s].data_ptr()
            io.out = outs[s].data_ptr()
            io.sel_chunk, io.sel_group = selc[s].data_ptr(), sels[s].data_ptr()
            io.cache = cache.c()
            dims = hga._Dims(w.B, cap, w.Hq, w.Hkv, w.D, 1)
            pc = hp.c()
            base = (ws.data_ptr() + 255) // 256 * 256
            st = hga.load().hga_forward(hga.DECODE, ctypes.byref(dims), ctypes.byref(pc),
                                        ctypes.byref(io), ctypes.c_void_p(base),
                                        ws.numel() - 256, hga._stream(None))
            assert st == 0

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run_steps()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    cache.lens.fill_(w.T)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_steps()
    cache.lens.fill_(w.T)
    graph.replay()
    torch.cuda.synchronize()
    assert (cache.lens == cap).all()
    p = oracle.Params.of(w)
    tol = TOL[w.dtype]
    for b in (3, 11):
        K = torch.cat([d["k_hist"][b], d["k_new"][:, b]], 0)[None].cpu()
        V = torch.cat([d["v_hist"][b], d["v_new"][:, b]], 0)[None].cpu()
        pos = torch.cat([d["pos_hist"][b], d["pos_new"][:, b]], 0)[None].cpu()
        steps = list(range(S))
        Q = np.zeros((1, cap, w.Hq, w.D))
        Q[0, w.T:] = d["q"][:, b].double().cpu().numpy()
        units = [(0, w.T + s) for s in steps]
        rr = oracle.hga(Q, K, V, pos, p, route_block=1, units=units, attend=False)
        ref = RouteRef(Q, K, pos, p, w.Hkv)
        sc, sg = selc[:, b].cpu().numpy(), sels[:, b].cpu().numpy()
        for i, (_, t) in enumerate(units):
            for h in range(w.Hkv):
                ok, _ = check_unit_selection(ref, 0, h, t, t + 1, t // 64, sc[t - w.T, h],
                                             sg[t - w.T, h], rr["sel_c"][i, h], rr["sel_g"][i, h])
                assert ok, f"routing mismatch b={b} t={t} h={h}"
        # 32 steps per sequence, 64 (sequence, step) outputs in all
        edges = [0, 1, 63, 64, 127, 128, 200, S - 1]
        sample = sorted(edges + [s for s in range(2, S - 1, 10) if s not in edges][:32 - len(edges)])
        assert len(sample) == 32
        u2 = [(0, w.T + s) for s in sample]
        force = np.stack([sg[s] for s in sample])
        orc = oracle.hga(Q, K, V, pos, p, route_block=1, units=u2, sel_g_force=force)
        O = outs[:, b].float().cpu().numpy()
        for s in sample:
            e = row_rel_err(O[s], orc["O"][0, w.T + s])
            assert e <= tol, f"decode output rel err {e} at b={b} step={s}"
        S_c, _ = oracle.build_summaries(K, pos, p)
        assert row_rel_err(_np(cache.s_chunk[b:b + 1]), S_c) < 2e-6


def test_decode_bounds_status_is_recorded(gpu_lib):
    """A sequence whose cache is already full is refused by the kernels' own
    index checks (before any access): the step leaves it untouched, records
    HGA_ERR_BOUNDS for hga_device_status, and the other sequences are served
    exactly as in a step without it."""
    w = QWEN.replace(B=2, Hq=8, Hkv=2)
    T_hist, cap = 640, 704
    d = make_decode_inputs(w, seed=3, T=T_hist, steps=1)
    dev = torch.device("cuda")
    hga = gpu_lib
    hp = _hp(hga, w)
    dt = d["k_hist"].dtype
    caches = []
    for _ in range(2):
        c = hga.KVCache(w.B, cap, w.Hkv, w.D, dt, hp, device=dev)
        hga.hga_fill_cache(d["k_hist"].to(dev), d["v_hist"].to(dev), d["pos_hist"].to(dev), c, hp)
        caches.append(c)
    assert hga.hga_device_status(clear=True) == 0
    caches[1].lens[0] = cap            # sequence 0 of the second cache: no room left
    args = (d["q"][0].to(dev), d["k_new"][0].to(dev), d["v_new"][0].to(dev),
            d["pos_new"][0].to(dev))
    good = hga.hga_forward_decode(*args, caches[0], hp)
    assert hga.hga_device_status(clear=True) == 0
    bad = hga.hga_forward_decode(*args, caches[1], hp)
    assert hga.hga_device_status(clear=False) == 5          # HGA_ERR_BOUNDS
    assert hga.hga_device_status(clear=True) == 5
    assert hga.hga_device_status(clear=True) == 0           # reset
    torch.cuda.synchronize()
    assert int(caches[1].lens[0]) == cap and int(caches[1].lens[1]) == T_hist + 1
    assert torch.equal(good["out"][1].view(torch.int16), bad["out"][1].view(torch.int16))
