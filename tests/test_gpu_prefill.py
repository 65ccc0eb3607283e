"""GPU parity of the prefill path (summaries, routing, attention) against the
CPU oracle, through the C ABI (via the thin Python binding).

Sizes: small enough for the oracle to finish in seconds, spanning several
tiles and ragged tails; plus the 32K Qwen3-shaped workload at full size in
the launch configuration the bench times, with every routed index set
compared and outputs on sampled blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.parity import TOL, RouteRef, check_unit_selection, row_rel_err
from workloads import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny_f32_prefill_1k"]
SMALLLM = WORKLOADS["smalllm40m_bf16_prefill_4k"]
QWEN = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"]

CASES = {
    "tiny_f32_1k": TINY,
    "f32_ragged_1000": TINY.replace(T=1000),
    "f32_F0_L0_gqa": TINY.replace(T=700, F=0, L=0, Hq=4, Hkv=2, K_c=3, K_g=5),
    "f32_gs8_D128": TINY.replace(T=832, g_s=8, D=128, Hq=8, Hkv=2, theta=1e6),
    "f32_gs64": TINY.replace(T=900, g_s=64, K_g=3),
    "f32_gs1": TINY.replace(T=512, g_s=1, K_g=40),
    "f32_T1": TINY.replace(T=1),
    "f32_T63": TINY.replace(T=63),
    "f32_T65": TINY.replace(T=65),
    "f32_full_budget": TINY.replace(T=640, K_c=64, K_g=256),
    "bf16_smalllm_2x1024": SMALLLM.replace(B=2, T=1024),
    "bf16_qwen_2048": QWEN.replace(T=2048),
    "bf16_qwen_ragged": QWEN.replace(T=64 * 20 + 33),
    "bf16_qwen_L0_F0": QWEN.replace(T=1280, F=0, L=0, K_c=5, K_g=9),
    # two sequences with a ragged last block: the output tiles of the first
    # sequence's last block must not reach into the second sequence
    "bf16_qwen_2x_ragged": QWEN.replace(B=2, T=64 * 9 + 17),
    # bf16 shapes the tensor-core kernel does not take (Hq/Hkv not a power of
    # two; groups shorter than its 8-token segments) run on the CUDA cores
    "bf16_G3_cuda_cores": QWEN.replace(T=64 * 12 + 5, Hq=6, Hkv=2, K_c=4, K_g=8),
    "bf16_gs4_cuda_cores": SMALLLM.replace(B=1, T=900, Hq=4, Hkv=4, g_s=4, K_g=24),
}


def _hp(w):
    import hierarchical_kv_routing_b200 as hga
    return hga.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                         rope_theta=w.theta)


def _np(t):
    return t.detach().float().cpu().numpy()


def run_and_check(hga, w, seed, units=None, sample_rows=None, pos_mod=None):
    q, k, v, pos, _ = make_prefill_inputs(w, seed=seed)
    if pos_mod:
        pos = (pos % pos_mod).contiguous()
    dev = torch.device("cuda")
    qd, kd, vd, pd = (x.to(dev) for x in (q, k, v, pos))
    hp = _hp(w)
    p = oracle.Params.of(w)
    tol = TOL[w.dtype]

    k_rot, s_c, s_g = hga.hga_build_summaries(kd, pd, hp)
    sel_c, sel_g = hga.hga_route(qd, pd, s_c, s_g, hp)
    out, lse = hga.hga_attend(qd, pd, k_rot, vd, sel_g, hp, want_lse=True)
    res = hga.hga_forward_prefill(qd, kd, vd, pd, hp, want_lse=True, want_sel=True)
    torch.cuda.synchronize()
    # the one-call path runs the same kernels (for bf16 with the rotated
    # queries handed from routing to attention): identical results
    bits = torch.int16 if w.dtype == "bf16" else torch.int32
    assert torch.equal(res["sel_chunk"], sel_c) and torch.equal(res["sel_group"], sel_g)
    assert torch.equal(res["out"].view(bits), out.view(bits))
    if w.dtype == "bf16":
        # the stage calls with the hand-off: the same bits again
        q_rot = torch.empty_like(qd)
        sc2, sg2 = hga.hga_route(qd, pd, s_c, s_g, hp, q_rot=q_rot)
        out2, lse2 = hga.hga_attend(qd, pd, k_rot, vd, sg2, hp, want_lse=True, q_rot=q_rot)
        torch.cuda.synchronize()
        assert torch.equal(sg2, sel_g) and torch.equal(out2.view(bits), out.view(bits))
        assert torch.equal(lse2, lse)

    # stage 1: K_rot and summaries
    ref = RouteRef(q, k, pos, p, w.Hkv)
    krot_ref = oracle.rope_rows(k, np.broadcast_to(_np(pd)[:, :, None], k.shape[:3]), w.theta)
    kr = _np(k_rot)
    ulp = 2.0 ** -8 if w.dtype == "bf16" else 2.0 ** -22
    assert np.all(np.abs(kr - krot_ref) <= ulp * np.abs(krot_ref) + 1e-6), "K_rot"
    for gpu, orc in ((s_c, ref.S_c), (s_g, ref.S_g)):
        if orc.size:
            assert row_rel_err(_np(gpu), orc) < 2e-6, "summaries"

    # stage 2: every routed set (all units), with the tie rule
    B, T = w.B, pos.shape[1]
    NB = (T + 63) // 64
    sc, sg = sel_c.cpu().numpy(), sel_g.cpu().numpy()
    all_units = [(b, u) for b in range(B) for u in range(NB)]
    rr = oracle.hga(q, k, v, pos, p, units=all_units, attend=False)
    tie_units = []
    for i, (b, u) in enumerate(all_units):
        for h in range(w.Hkv):
            ok, tie = check_unit_selection(ref, b, h, 64 * u, min(T, 64 * u + 64), u,
                                           sc[b, u, h], sg[b, u, h], rr["sel_c"][i, h],
                                           rr["sel_g"][i, h])
            assert ok, f"routing mismatch at b={b} block={u} h={h}"
            if tie:
                tie_units.append((b, u))

    # stage 3: outputs on the checked units
    units = all_units if units is None else units
    force = np.stack([sg[b, u] for (b, u) in units])
    orc = oracle.hga(q, k, v, pos, p, units=units, sel_g_force=force)
    O = _np(out)
    L = _np(lse)
    for (b, u) in units:
        sl = slice(64 * u, min(T, 64 * u + 64))
        e = row_rel_err(O[b, sl], orc["O"][b, sl])
        assert e <= tol, f"output rel err {e} at b={b} block={u}"
        le = np.abs(L[b, :, sl] - orc["LSE"][b, :, sl]).max()
        assert le <= (1e-5 if w.dtype == "f32" else 2e-2) * max(1.0, np.abs(orc["LSE"][b, :, sl]).max()), "lse"
    return {"tie_units": tie_units}


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_parity(gpu_lib, name):
    run_and_check(gpu_lib, CASES[name], seed=7)


def test_full_budget_is_dense(gpu_lib):
    w = TINY.replace(T=640, K_c=64, K_g=256, Hq=4, Hkv=2)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=3)
    dev = torch.device("cuda")
    res = gpu_lib.hga_forward_prefill(*(x.to(dev) for x in (q, k, v, pos)), _hp(w))
    O, _ = oracle.dense(q, k, v, pos, w.theta)
    assert row_rel_err(_np(res["out"]), O) <= 1e-5


@pytest.mark.slow
def test_qwen_32k_full_size(gpu_lib):
    """The 32K Qwen3-shaped prefill exactly as the bench runs it: every
    routed set checked; outputs on sampled blocks (first F+L+2, a spread
    through the middle and the last)."""
    w = QWEN
    NB = w.T // 64
    blocks = list(range(0, w.F + w.L + 2)) + list(range(w.F + w.L + 3, NB - 1, 9)) + [NB - 1]
    assert len(blocks) >= 64
    run_and_check(gpu_lib, w, seed=11, units=[(0, u) for u in blocks])


def test_exact_token_chunk_variant(gpu_lib):
    """The exact-token chunk variant (groups off: every group of each routed
    chunk opened, page section 3, routing policy) is K_g = K_c * C / g_s: the
    routed groups are exactly the groups of the routed chunks, and outputs
    match the oracle."""
    w = QWEN.replace(T=64 * 40 + 17, K_c=6, K_g=6 * 4)
    run_and_check(gpu_lib, w, seed=21)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=21)
    dev = torch.device("cuda")
    res = gpu_lib.hga_forward_prefill(*(x.to(dev) for x in (q, k, v, pos)), _hp(w), want_sel=True)
    sc, sg = res["sel_chunk"].cpu().numpy(), res["sel_group"].cpu().numpy()
    gpc = w.C // w.g_s
    for blk in range(sc.shape[1]):
        for h in range(w.Hkv):
            chunks = sc[0, blk, h][sc[0, blk, h] >= 0]
            groups = sg[0, blk, h][sg[0, blk, h] >= 0]
            assert sorted(groups.tolist()) == sorted((chunks[:, None] * gpc + np.arange(gpc)).ravel().tolist())


def test_attend_rejects_unaligned_output(gpu_lib):
    """Tensor pointers must be 16-byte aligned (the output leaves by tensor
    stores): another base is refused before any launch."""
    hga = gpu_lib
    w = CASES["bf16_qwen_2x_ragged"]
    q, k, v, pos, _ = make_prefill_inputs(w, seed=3)
    dev = torch.device("cuda")
    qd, kd, vd, pd = (x.to(dev) for x in (q, k, v, pos))
    hp = _hp(w)
    k_rot, s_c, s_g = hga.hga_build_summaries(kd, pd, hp)
    _, sel_g = hga.hga_route(qd, pd, s_c, s_g, hp)
    raw = torch.zeros((qd.numel() + 1,), dtype=qd.dtype, device=dev)
    shifted = raw[1:].view(qd.shape)
    assert shifted.data_ptr() % 16 != 0
    with pytest.raises(hga.HGAError, match="invalid argument"):
        hga.hga_attend(qd, pd, k_rot, vd, sel_g, hp, out=shifted)
    torch.cuda.synchronize()
    assert not raw.any()


@pytest.mark.parametrize("name,mod", [("f32_ragged_1000", 300), ("bf16_qwen_ragged", 1000)])
def test_prefill_wrapped_positions(gpu_lib, name, mod):
    """Positions taken modulo a period shorter than the sequence (the pages'
    position-mod-65536 variant, at a period the oracle can check quickly):
    RoPE and the summaries' mean positions use the given positions, while
    causality and the chunk structure follow the token index."""
    run_and_check(gpu_lib, CASES[name], seed=17, pos_mod=mod)


@pytest.mark.slow
def test_smalllm_4k_full_size(gpu_lib):
    """The SmallLM-40M-shaped prefill (8 sequences x 4096 tokens, 8 heads,
    MHA, D=64) exactly as the bench times it: every routed set of every
    sequence checked; outputs on 64 sampled (sequence, block) pairs that
    include the first F+L+2 blocks and the last block."""
    w = SMALLLM
    NB = w.T // 64
    first = list(range(0, w.F + w.L + 2))
    units = [(0, u) for u in first] + [(7, NB - 1)]
    for b in range(w.B):
        for u in (w.F + w.L + 2 + 7 * b, 31 + b, 40 + 3 * b, 50 + b, NB - 1 - b, 13 + 5 * b,
                  22 + 2 * b, 57 - b):
            if (b, u) not in units:
                units.append((b, u))
    units = units[:max(64, len(first) + 1)]
    assert len(units) >= 64 and (7, NB - 1) in units
    run_and_check(gpu_lib, w, seed=13, units=units)
