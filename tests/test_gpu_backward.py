"""GPU parity of the backward of routed attention (hga_attend_backward)
against the CPU oracle's or_hga_backward, through the C ABI.

The forward runs first (summaries, routing, attention with LSE); the
backward then gets the forward's routed groups, output and LSE and a seeded
d_out.  The oracle differentiates the same attention in fp64 with the same
routed groups (routing is a discrete choice, held fixed), so the comparison
is of dq, dk and dv alone.  Bars: per row (the D values of one query or key
row), max|gpu - ref| / max(max|ref_row|, 1% of the largest ref row) within
1e-5 for fp32 inputs (the CUDA-core path: fp32 arithmetic, atomic sums) and
2e-2 for bf16 inputs (the tensor-core path: bf16 operands, P and dS rounded
to bf16 for the products, fp32 accumulation).  The 1% floor keeps rows that
are nearly zero (a key that few queries see, with small weights) from
turning an absolute rounding error into a large relative one.
"""
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


def grad_err(gpu, ref):
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    num = np.abs(g - r).max(-1)
    mag = np.abs(r).max(-1)
    den = np.maximum(mag, 0.01 * max(float(mag.max()), 1e-30))
    return float((num / den).max()) if num.size else 0.0


def run_backward(hga, w, seed, dO_blocks=None):
    """Forward + backward on the GPU; returns (gpu grads, oracle grads)."""
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
    dq, dk, dv = hga.hga_attend_backward(qd, pd, k_rot, vd, sel_g, out, lse, gd, hp)
    torch.cuda.synchronize()
    assert hga.hga_device_status() == 0
    ref = oracle.hga_backward(q, k, v, pos, dO, oracle.Params.of(w), sel_g.cpu().numpy())
    return tuple(x.cpu().numpy() for x in (dq, dk, dv)), ref


@pytest.mark.parametrize("name", list(CASES))
def test_backward_parity(gpu_lib, name):
    w = CASES[name]
    got, ref = run_backward(gpu_lib, w, seed=31)
    tol = TOL[w.dtype]
    for label, a, b in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(a).all(), label
        e = grad_err(a, b)
        assert e <= tol, f"{label} rel err {e} > {tol}"


def test_backward_full_budget_equals_dense_gradients(gpu_lib):
    """With every middle chunk and group routed, routed attention is dense
    causal attention (Table 7's check), so its gradients are dense
    attention's: the oracle's, taken with the full-budget routed set."""
    w = QWEN.replace(T=576, K_c=64, K_g=256, Hq=8, Hkv=2)
    got, ref = run_backward(gpu_lib, w, seed=33)
    for a, b in zip(got, ref):
        assert grad_err(a, b) <= TOL["bf16"]


def test_backward_twice_is_stable(gpu_lib):
    """Two calls in a row on the same inputs: dq is bit-identical (its rows
    are owned by one CTA each); dk and dv are sums formed by atomic additions
    and agree to rounding."""
    w = QWEN.replace(T=1024)
    dev = torch.device("cuda")
    q, k, v, pos, _ = make_prefill_inputs(w, seed=35, device=dev)
    hp = _hp(gpu_lib, w)
    dO = torch.randn(q.shape, generator=torch.Generator(device=dev).manual_seed(1), device=dev,
                     dtype=torch.float32).to(q.dtype)
    k_rot, s_c, s_g = gpu_lib.hga_build_summaries(k, pos, hp)
    _, sel_g = gpu_lib.hga_route(q, pos, s_c, s_g, hp)
    out, lse = gpu_lib.hga_attend(q, pos, k_rot, v, sel_g, hp, want_lse=True)
    a = gpu_lib.hga_attend_backward(q, pos, k_rot, v, sel_g, out, lse, dO, hp)
    b = gpu_lib.hga_attend_backward(q, pos, k_rot, v, sel_g, out, lse, dO, hp)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    for x, y in zip(a[1:], b[1:]):
        assert (x - y).abs().max().item() <= 1e-5 * max(1.0, x.abs().max().item())


@pytest.mark.slow
def test_backward_qwen_32k_full_size(gpu_lib):
    """The 32K Qwen3-shaped workload at full size, with d_out nonzero on 64
    sampled query blocks (the first F+L+2, a spread through the middle and
    the last) and zero elsewhere: every element of dq, dk and dv is compared
    with the oracle, which skips rows whose d_out is zero (exactly: they add
    nothing to any gradient)."""
    w = QWEN
    NB = w.T // 64
    blocks = list(range(0, w.F + w.L + 2)) + list(range(w.F + w.L + 3, NB - 1, 10)) + [NB - 1]
    assert len(blocks) >= 60
    got, ref = run_backward(gpu_lib, w, seed=37, dO_blocks=blocks)
    for label, a, b in zip(("dq", "dk", "dv"), got, ref):
        e = grad_err(a, b)
        assert e <= TOL["bf16"], f"{label} rel err {e}"
