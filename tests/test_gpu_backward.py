"""GPU parity of the backward of routed attention (hga_attend_backward)
against the CPU oracle's or_hga_backward, through the C ABI.

The forward runs first (summaries, routing, attention with LSE); the
backward then gets the forward's routed groups and LSE and a seeded d_out.
The oracle differentiates the same attention in fp64 with the same routed
groups (routing is a discrete choice, held fixed), so the comparison is of
dq, dk and dv alone.

The bar.  The pages fix a tolerance for outputs only.  A gradient entry is a
sum of terms of both signs that can cancel (the dS_ij of one row sum to
zero), so a relative bar on the entry itself is not met by any rounding of
the terms; the bar here is relative to the magnitude of the terms, the usual
error bound of a sum (the routing tie rule scales the same way):
  dq_i: |err| <= tol * max_d sum_j P_ij (|dP_ij| + |Delta_i|) |k~_jd| / sqrt(D)
  dk_j: |err| <= tol * max_d sum_i P_ij (|dP_ij| + |Delta_i|) |q~_id| / sqrt(D)
  dv_j: |err| <= tol * max_d sum_i P_ij |dO_id|
with tol = 1e-5 for fp32 inputs (CUDA cores, fp32 arithmetic) and 2e-2 for
bf16 inputs (tensor cores: bf16 operands, P and dS rounded to bf16 for the
products, fp32 accumulation), the output tolerances of the forward.  The
magnitudes are computed here from exact fp64 rotations; the expected values
come from the oracle alone.  Each tensor must also be within tol of the
oracle in the Frobenius norm.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_prefill_inputs

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny_f32_prefill_1k"]
SMALLLM = WORKLOADS["smalllm40m_bf16_prefill_4k"]
QWEN = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"]
TOL = {"f32": 1e-5, "bf16": 2e-2}

CASES = {
    "f32_tiny_1k": TINY,
    "f32_ragged_gqa": TINY.replace(T=700, Hq=4, Hkv=2),
    "f32_F0_L0": TINY.replace(T=650, F=0, L=0, K_c=3, K_g=5),
    "f32_gs8_D128": TINY.replace(T=576, g_s=8, D=128, Hq=8, Hkv=2, theta=1e6),
    "bf16_qwen_2048": QWEN.replace(T=2048),
    "bf16_qwen_ragged": QWEN.replace(T=64 * 20 + 33),
    "bf16_qwen_L0_F0": QWEN.replace(T=1280, F=0, L=0, K_c=5, K_g=9),
    "bf16_qwen_G16": QWEN.replace(T=1024 + 17, Hq=32, Hkv=2),
    "bf16_qwen_G1": QWEN.replace(T=960, Hq=4, Hkv=4),
    "bf16_smalllm_2x1024": SMALLLM.replace(B=2, T=1024),
    "bf16_smalllm_ragged": SMALLLM.replace(B=2, T=64 * 9 + 5),
    "bf16_full_budget": QWEN.replace(T=640, K_c=64, K_g=256),
    # bf16 shapes the tensor-core kernels do not take: CUDA cores
    "bf16_G3_cuda_cores": QWEN.replace(T=64 * 12 + 5, Hq=6, Hkv=2, K_c=4, K_g=8),
    "bf16_gs4_cuda_cores": SMALLLM.replace(B=1, T=900, Hq=4, Hkv=4, g_s=4, K_g=24),
}


def _hp(hga, w):
    return hga.HGAParams(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g,
                         rope_theta=w.theta)


def term_scales(q, k, v, pos, dO, p, sel_g, tokens=None):
    """Per-row magnitude of the terms that form each gradient entry (see the
    module docstring): (Mq [B,T,Hq], Mk [B,T,Hkv], Mv [B,T,Hkv]), in fp64 on
    the GPU.  tokens: the query tokens whose d_out is nonzero (default all;
    the others add nothing to any gradient)."""
    dev = torch.device("cuda")
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    G, H = Hq // Hkv, D // 2
    rows = list(range(T)) if tokens is None else sorted(tokens)
    ridx = torch.tensor(rows, device=dev)
    om = torch.tensor(p.theta ** (-2.0 * np.arange(H) / D), dtype=torch.float64, device=dev)

    def rope(x, pp):                      # x [n, heads, D], pp [n]
        a = pp.double()[:, None] * om
        c, s_ = torch.cos(a)[:, None, :], torch.sin(a)[:, None, :]
        return torch.cat([x[..., :H] * c - x[..., H:] * s_, x[..., H:] * c + x[..., :H] * s_], -1)

    Mq = torch.zeros(B, T, Hq, dtype=torch.float64, device=dev)
    Mk = torch.zeros(B, T, Hkv, dtype=torch.float64, device=dev)
    Mv = torch.zeros(B, T, Hkv, dtype=torch.float64, device=dev)
    sg = np.asarray(sel_g)
    for b in range(B):
        pb = torch.as_tensor(np.asarray(pos)[b], device=dev)
        qt = rope(torch.as_tensor(np.asarray(q[b], np.float64), device=dev)[ridx], pb[ridx])
        kt = rope(torch.as_tensor(np.asarray(k[b], np.float64), device=dev), pb)
        vb = torch.as_tensor(np.asarray(v[b], np.float64), device=dev)
        gb = torch.as_tensor(np.asarray(dO[b], np.float64), device=dev)[ridx]
        for h in range(Hkv):
            mask = torch.from_numpy(np.stack(
                [oracle.visible_mark(i // p.C, i, T, sg[b, i // p.C, h], p) for i in rows])).to(dev)
            ak = torch.zeros(T, D, dtype=torch.float64, device=dev)
            av = torch.zeros(T, D, dtype=torch.float64, device=dev)
            for hq in range(h * G, (h + 1) * G):
                s_ = (qt[:, hq] @ kt[:, h].T / math.sqrt(D)).masked_fill(~mask, float("-inf"))
                P = torch.softmax(s_, -1)
                dp = gb[:, hq] @ vb[:, h].T
                delta = (P * dp).sum(-1, keepdim=True)
                A = P * (dp.abs() + delta.abs())
                Mq[b, ridx, hq] = (A @ kt[:, h].abs()).amax(-1) / math.sqrt(D)
                ak += A.T @ qt[:, hq].abs() / math.sqrt(D)
                av += P.T @ gb[:, hq].abs()
            Mk[b, :, h] = ak.amax(-1)
            Mv[b, :, h] = av.amax(-1)
    return Mq.cpu().numpy(), Mk.cpu().numpy(), Mv.cpu().numpy()


def check_grads(got, ref, scales, tol):
    for label, a, b, m in zip(("dq", "dk", "dv"), got, ref, scales):
        assert np.isfinite(a).all(), label
        err = np.abs(np.asarray(a, np.float64) - b).max(-1)
        worst = float((err / np.maximum(m, 1e-300)).max())
        assert np.all(err <= tol * m + 1e-30), f"{label}: error / term scale {worst} > {tol}"
        nw = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
        assert nw <= tol, f"{label}: normwise rel err {nw} > {tol}"


def run_backward(hga, w, seed, dO_blocks=None):
    """Forward + backward on the GPU; returns (gpu grads, oracle grads, term
    scales)."""
    dev = torch.device("cuda")
    q, k, v, pos, _ = make_prefill_inputs(w, seed=seed)
    dtype = q.dtype
    g = torch.Generator().manual_seed(seed + 1000)
    dO = torch.randn(q.shape, generator=g, dtype=torch.float32).to(dtype)
    if dO_blocks is not None:
        keep = torch.zeros(w.T, dtype=torch.bool)
        for blk in dO_blocks:
            keep[64 * blk:64 * blk + 64] = True
        dO[:, ~keep] = 0
    qd, kd, vd, pd, gd = (x.to(dev) for x in (q, k, v, pos, dO))
    hp = _hp(hga, w)
    k_rot, s_c, s_g = hga.hga_build_summaries(kd, pd, hp)
    sel_c, sel_g = hga.hga_route(qd, pd, s_c, s_g, hp)
    out, lse = hga.hga_attend(qd, pd, k_rot, vd, sel_g, hp, want_lse=True)
    dq, dk, dv = hga.hga_attend_backward(qd, pd, k_rot, vd, sel_g, lse, gd, hp)
    torch.cuda.synchronize()
    assert hga.hga_device_status() == 0
    p = oracle.Params.of(w)
    sg = sel_g.cpu().numpy()
    ref = oracle.hga_backward(q, k, v, pos, dO, p, sg)
    tokens = None
    if dO_blocks is not None:
        tokens = [t for blk in dO_blocks for t in range(64 * blk, min(w.T, 64 * blk + 64))]
    scales = term_scales(q.float().numpy(), k.float().numpy(), v.float().numpy(), pos.numpy(),
                         dO.float().numpy(), p, sg, tokens)
    return tuple(x.cpu().numpy() for x in (dq, dk, dv)), ref, scales


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(gpu_lib, name):
    w = CASES[name]
    got, ref, scales = run_backward(gpu_lib, w, seed=31)
    check_grads(got, ref, scales, TOL[w.dtype])


def test_backward_full_budget_equals_dense_gradients(gpu_lib):
    """With every middle chunk and group routed, routed attention is dense
    causal attention (Table 7's check), so its gradients are dense
    attention's: compared with the oracle's dense-causal gradients, taken as
    the routed backward over the full budget (pinned to autograd of dense
    attention on the CPU)."""
    w = QWEN.replace(T=576, K_c=64, K_g=256, Hq=8, Hkv=2)
    got, ref, scales = run_backward(gpu_lib, w, seed=33)
    check_grads(got, ref, scales, TOL["bf16"])


def test_backward_twice_is_stable(gpu_lib):
    """Two calls in a row on the same inputs, and a third given the rotated
    queries from routing: dq is bit-identical (its rows are owned by one CTA
    each); dk and dv are sums formed by atomic additions and agree to
    rounding."""
    w = QWEN.replace(T=1024)
    dev = torch.device("cuda")
    q, k, v, pos, _ = make_prefill_inputs(w, seed=35, device=dev)
    hp = _hp(gpu_lib, w)
    dO = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(1), device=dev,
                     dtype=torch.float32).to(q.dtype)
    k_rot, s_c, s_g = gpu_lib.hga_build_summaries(k, pos, hp)
    _, sel_g = gpu_lib.hga_route(q, pos, s_c, s_g, hp)
    out, lse = gpu_lib.hga_attend(q, pos, k_rot, v, sel_g, hp, want_lse=True)
    a = gpu_lib.hga_attend_backward(q, pos, k_rot, v, sel_g, lse, dO, hp)
    b = gpu_lib.hga_attend_backward(q, pos, k_rot, v, sel_g, lse, dO, hp)
    # with the rotated queries the forward's routing wrote: the same dq bits
    q_rot = torch.empty_like(q)
    gpu_lib.hga_route(q, pos, s_c, s_g, hp, q_rot=q_rot)
    c = gpu_lib.hga_attend_backward(q, pos, k_rot, v, sel_g, lse, dO, hp, q_rot=q_rot)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[0], c[0])
    for x, y, z in zip(a[1:], b[1:], c[1:]):
        assert (x - y).abs().max().item() <= 1e-5 * max(1.0, x.abs().max().item())
        assert (x - z).abs().max().item() <= 1e-5 * max(1.0, x.abs().max().item())


@pytest.mark.slow
def test_backward_qwen_32k_full_size(gpu_lib):
    """The 32K Qwen3-shaped workload at full size, with d_out nonzero on 63
    sampled query blocks (the first F+L+2, a spread through the middle and
    the last) and zero elsewhere: every element of dq, dk and dv is compared
    with the oracle, which skips rows whose d_out is zero (exactly: they add
    nothing to any gradient)."""
    w = QWEN
    NB = w.T // 64
    blocks = list(range(0, w.F + w.L + 2)) + list(range(w.F + w.L + 3, NB - 1, 10)) + [NB - 1]
    assert len(blocks) >= 60
    got, ref, scales = run_backward(gpu_lib, w, seed=37, dO_blocks=blocks)
    check_grads(got, ref, scales, TOL["bf16"])
