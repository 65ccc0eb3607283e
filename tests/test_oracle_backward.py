"""Pins of the oracle's backward pass of routed attention.

Method page: HGA paper review, Tab. 8 "Training and Prefill Speed" (training
through HGA attention) and Sec. 5.9 "Fine-tuning Stability" (QK fine-tuning
through the routed attention in exact-token mode).  The page prints no
formula for the gradients; the oracle differentiates eq. (1) restricted to
each query's visible set with the routed groups held fixed.  These tests pin
it to things other than its own derivation: automatic differentiation of the
same attention written with library ops (RoPE as a complex product, softmax
under a boolean mask), central differences of the oracle's forward pass, the
sum rules of a softmax gradient, and position-shift invariance.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_prefill_inputs


def _params(**kw):
    d = dict(C=64, g_s=16, F=2, L=2, K_c=4, K_g=8, theta=1e4, hf_wavelength=0.0)
    d.update(kw)
    return oracle.Params(**d)


def _autograd(Q, K, V, pos, theta, mask, dO):
    """Gradients of sum(dO * O) for O = softmax attention under `mask`
    [B, Hq, T, T], RoPE written as multiplication by exp(i p w) of the complex
    pairs x_i + i x_{i+D/2}, GQA by repeating KV heads."""
    Q, K, V = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    B, T, Hq, D = Q.shape
    Hkv, H = K.shape[2], D // 2
    G = Hq // Hkv
    w = theta ** (-2.0 * torch.arange(H, dtype=torch.float64) / D)
    ang = torch.tensor(pos, dtype=torch.float64)[..., None] * w
    rot = torch.polar(torch.ones_like(ang), ang)[:, :, None, :]

    def rope(x):
        z = torch.complex(x[..., :H], x[..., H:]) * rot
        return torch.cat([z.real, z.imag], -1)

    q = rope(Q)
    k = rope(K).repeat_interleave(G, dim=2)
    v = V.repeat_interleave(G, dim=2)
    s = torch.einsum("bihd,bjhd->bhij", q, k) / math.sqrt(D)
    s = s.masked_fill(~torch.from_numpy(mask), float("-inf"))
    O = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, -1), v)
    (O * torch.from_numpy(dO)).sum().backward()
    return Q.grad.numpy(), K.grad.numpy(), V.grad.numpy()


def _routed_mask(sel_g, B, T, Hq, Hkv, p):
    mask = np.zeros((B, Hq, T, T), bool)
    G = Hq // Hkv
    for b in range(B):
        for i in range(T):
            c = i // p.C
            for h in range(Hkv):
                mask[b, h * G:(h + 1) * G, i] = oracle.visible_mark(c, i, T, sel_g[b, c, h], p)
    return mask


def _routed(Q, K, V, pos, p):
    """The oracle's own routed groups, as [B, NB, Hkv, K_g]."""
    B, T = Q.shape[:2]
    NB = (T + p.C - 1) // p.C
    return oracle.hga(Q, K, V, pos, p, attend=False)["sel_g"].reshape(B, NB, K.shape[2], p.K_g)


@pytest.mark.parametrize("T,F,L,g_s,Hq,Hkv", [(200, 2, 2, 16, 4, 2), (64 * 4 + 5, 1, 0, 8, 3, 1)])
def test_full_budget_backward_equals_dense_autograd(T, F, L, g_s, Hq, Hkv):
    # every middle chunk and group routed: the gradients are dense causal attention's
    rng = np.random.default_rng(T + Hq)
    B, D = 2, 32
    Q = rng.standard_normal((B, T, Hq, D))
    K = rng.standard_normal((B, T, Hkv, D))
    V = rng.standard_normal((B, T, Hkv, D))
    dO = rng.standard_normal((B, T, Hq, D))
    pos = np.tile(np.arange(T, dtype=np.int32), (B, 1))
    nc = T // 64 + 1
    p = _params(F=F, L=L, g_s=g_s, K_c=nc, K_g=nc * (64 // g_s))
    got = oracle.hga_backward(Q, K, V, pos, dO, p, _routed(Q, K, V, pos, p))
    causal = np.broadcast_to(np.tril(np.ones((T, T), bool)), (B, Hq, T, T)).copy()
    want = _autograd(Q, K, V, pos, p.theta, causal, dO)
    for g, w in zip(got, want):
        np.testing.assert_allclose(g, w, atol=1e-10, rtol=0)


def test_routed_backward_equals_masked_autograd():
    # a sparse routed set (the tiny workload's own routing): autograd under its mask
    w = WORKLOADS["tiny_f32_prefill_1k"]
    q, k, v, pos, _ = make_prefill_inputs(w, seed=5)
    q, k, v, pos = q.numpy(), k.numpy(), v.numpy(), pos.numpy()
    p = oracle.Params.of(w)
    rng = np.random.default_rng(6)
    dO = rng.standard_normal(q.shape)
    sel = _routed(q, k, v, pos, p)
    mask = _routed_mask(sel, w.B, w.T, w.Hq, w.Hkv, p)
    assert mask.sum() < 0.8 * np.tril(np.ones((w.T, w.T))).sum() * w.Hq   # really sparse
    got = oracle.hga_backward(q, k, v, pos, dO, p, sel)
    want = _autograd(q, k, v, pos, p.theta, mask, dO)
    for g, w_ in zip(got, want):
        np.testing.assert_allclose(g, w_, atol=1e-10, rtol=0)


def test_backward_matches_central_differences_of_forward():
    # d/dx of L = sum(dO * O) with the routed groups fixed, by central
    # differences of the oracle's forward pass at sampled coordinates
    rng = np.random.default_rng(7)
    B, T, Hq, Hkv, D = 1, 64 * 6, 2, 1, 16
    p = _params(F=1, L=1, K_c=2, K_g=3, theta=1e4)
    Q = rng.standard_normal((B, T, Hq, D))
    K = rng.standard_normal((B, T, Hkv, D))
    V = rng.standard_normal((B, T, Hkv, D))
    dO = rng.standard_normal((B, T, Hq, D))
    pos = (np.arange(T, dtype=np.int32) * 3 + 11)[None]
    sel = _routed(Q, K, V, pos, p)
    assert (sel >= 0).sum() > 0
    force = sel.reshape(-1, Hkv, p.K_g)
    dQ, dK, dV = oracle.hga_backward(Q, K, V, pos, dO, p, sel)

    def loss(Q_, K_, V_):
        return float((oracle.hga(Q_, K_, V_, pos, p, sel_g_force=force)["O"] * dO).sum())

    eps = 1e-5
    for name, X, grad in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in X.shape)
            # keys late in the sequence see few queries: sample the whole range
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += eps
            Xm[idx] -= eps
            args_p = {"Q": (Xp, K, V), "K": (Q, Xp, V), "V": (Q, K, Xp)}[name]
            args_m = {"Q": (Xm, K, V), "K": (Q, Xm, V), "V": (Q, K, Xm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx, fd, grad[idx])


def test_backward_sum_rules():
    # each query row's softmax weights sum to one, and its score gradients
    # sum to zero: sum_j dV_j = sum of dO over the KV head's query rows, and
    # sum_j R_{p_j}(dK_j) = 0 (the rotated key gradients cancel)
    w = WORKLOADS["tiny_f32_prefill_1k"].replace(T=448, Hq=4, Hkv=2)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=8)
    q, k, v, pos = q.numpy(), k.numpy(), v.numpy(), pos.numpy()
    p = oracle.Params.of(w)
    dO = np.random.default_rng(9).standard_normal(q.shape)
    dQ, dK, dV = oracle.hga_backward(q, k, v, pos, dO, p, _routed(q, k, v, pos, p))
    G = w.Hq // w.Hkv
    for h in range(w.Hkv):
        np.testing.assert_allclose(dV[:, :, h].sum(axis=1),
                                   dO[:, :, h * G:(h + 1) * G].sum(axis=(1, 2)), atol=1e-10)
        kr = oracle.rope_rows(dK[0, :, h], pos[0].astype(np.float64), w.theta)
        assert np.abs(kr.sum(axis=0)).max() < 1e-10 * max(1.0, np.abs(dK).max() * w.T)


def test_backward_constant_values_give_no_score_gradient():
    # with every v_j equal, O = v whatever the weights: dQ = dK = 0
    w = WORKLOADS["tiny_f32_prefill_1k"].replace(T=320)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=10)
    q, k, pos = q.numpy(), k.numpy(), pos.numpy()
    v = np.broadcast_to(np.random.default_rng(11).standard_normal(w.D), k.shape).copy()
    p = oracle.Params.of(w)
    dO = np.random.default_rng(12).standard_normal(q.shape)
    dQ, dK, dV = oracle.hga_backward(q, k, v, pos, dO, p, _routed(q, k, v, pos, p))
    assert np.abs(dQ).max() < 1e-12 and np.abs(dK).max() < 1e-12
    assert np.abs(dV).max() > 0.1


def test_backward_is_invariant_to_a_position_shift():
    # scores depend on position differences only, so the forward output and
    # all three raw-input gradients are unchanged when every position moves
    # by the same amount (a sign slip in the adjoint rotation breaks this)
    w = WORKLOADS["tiny_f32_prefill_1k"].replace(T=384, Hq=4, Hkv=2)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=13)
    q, k, v, pos = q.numpy(), k.numpy(), v.numpy(), pos.numpy()
    p = oracle.Params.of(w)
    dO = np.random.default_rng(14).standard_normal(q.shape)
    sel = _routed(q, k, v, pos, p)
    base = oracle.hga_backward(q, k, v, pos, dO, p, sel)
    for delta in (1, 977, 65536):
        moved = oracle.hga_backward(q, k, v, pos + delta, dO, p, sel)
        for a, b in zip(base, moved):
            np.testing.assert_allclose(a, b, atol=1e-9 * max(1.0, np.abs(a).max()), rtol=0)


def test_backward_with_dO_zero_outside_sampled_blocks_equals_masked_autograd():
    # dO nonzero on a few query blocks only (how the full-size GPU test
    # samples): the oracle skips the other rows, and its gradients still equal
    # automatic differentiation of the whole masked attention with that dO
    w = WORKLOADS["tiny_f32_prefill_1k"].replace(T=64 * 7 + 9, Hq=4, Hkv=2)
    q, k, v, pos, _ = make_prefill_inputs(w, seed=15)
    q, k, v, pos = q.numpy(), k.numpy(), v.numpy(), pos.numpy()
    p = oracle.Params.of(w)
    dO = np.random.default_rng(16).standard_normal(q.shape)
    keep = np.zeros(w.T, bool)
    for blk in (0, 3, 7):
        keep[64 * blk:64 * blk + 64] = True
    dO[:, ~keep] = 0.0
    dO[:, 64 * 3 + 5, 1] = 0.0           # one zero row inside a kept block
    sel = _routed(q, k, v, pos, p)
    got = oracle.hga_backward(q, k, v, pos, dO, p, sel)
    want = _autograd(q, k, v, pos, p.theta, _routed_mask(sel, w.B, w.T, w.Hq, w.Hkv, p), dO)
    for g, w_ in zip(got, want):
        np.testing.assert_allclose(g, w_, atol=1e-10, rtol=0)
    assert np.abs(got[0][:, ~keep]).max() == 0.0
