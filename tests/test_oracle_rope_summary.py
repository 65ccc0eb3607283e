"""Pins of the oracle's RoPE and mixed-RoPE summaries against facts that do
not come from the oracle itself: complex rotation, closed forms, the
method's special cases (g_s = 1; identical keys) and linearity.

Method page: HGA paper review, section 3, "Mixed-RoPE Routing Summaries".
"""
import math

import numpy as np
import pytest

import oracle


def _complex_rotate(x, p, theta):
    """Rotate-half pairs as complex numbers z_i = x_i + i x_{i+D/2} times
    e^{i p omega_i}; an independent route to the same rotation."""
    D = x.shape[-1]
    h = D // 2
    om = theta ** (-np.arange(h) * 2.0 / D)
    z = (x[..., :h] + 1j * x[..., h:]) * np.exp(1j * np.asarray(p)[..., None] * om)
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("D,theta", [(64, 1e4), (128, 1e6), (8, 10.0)])
def test_rope_matches_complex_rotation(D, theta):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((50, D))
    p = rng.integers(0, 70000, 50).astype(np.float64)
    got = oracle.rope_rows(x, p, theta)
    np.testing.assert_allclose(got, _complex_rotate(x, p, theta), rtol=0, atol=1e-9)


def test_rope_quarter_turn_and_identity():
    # omega_0 = 1, so position pi/2 turns pair 0 by exactly a quarter:
    # (x_0, x_h) -> (-x_h, x_0); position 0 is the identity.
    x = np.arange(1.0, 9.0)[None, :]
    y = oracle.rope_rows(x, np.array([math.pi / 2]), 1e4)
    assert abs(y[0, 0] - (-x[0, 4])) < 1e-12 and abs(y[0, 4] - x[0, 0]) < 1e-12
    np.testing.assert_array_equal(oracle.rope_rows(x, np.array([0.0]), 1e4), x)


def test_rope_relative_position_property():
    # <R_p q, R_s k> depends on p - s only; norm per pair is kept.
    rng = np.random.default_rng(1)
    D = 128
    q, k = rng.standard_normal((2, 1, D))
    for p, s, d in [(5, 3, 1000), (70000, 12, -11), (0, 0, 65535)]:
        a = (oracle.rope_rows(q, [p], 1e6) * oracle.rope_rows(k, [s], 1e6)).sum()
        b = (oracle.rope_rows(q, [p + d], 1e6) * oracle.rope_rows(k, [s + d], 1e6)).sum()
        assert abs(a - b) < 1e-9 * np.abs(q).sum() * np.abs(k).sum()
    y = oracle.rope_rows(q, [12345], 1e6)
    h = D // 2
    np.testing.assert_allclose(y[0, :h] ** 2 + y[0, h:] ** 2, q[0, :h] ** 2 + q[0, h:] ** 2,
                               rtol=1e-12)


@pytest.mark.parametrize("D,theta,expect", [(64, 1e4, 9), (128, 1e6, 11), (128, 1e4, 17)])
def test_high_pair_split_closed_form(D, theta, expect):
    # 2 pi / omega_i < C  <=>  i < (D / 2) ln(C / 2 pi) / ln theta
    hi = oracle.pair_is_high(D, theta, 0.0, 64)
    bound = (D / 2.0) * math.log(64 / (2 * math.pi)) / math.log(theta)
    assert hi.sum() == expect == math.ceil(bound)
    assert hi[: expect].all() and not hi[expect:].any()   # the fast pairs are the first ones
    assert oracle.pair_is_high(D, theta, math.inf, 64).all()
    assert not oracle.pair_is_high(D, theta, 1e-9, 64).any()


def _params(**kw):
    d = dict(C=64, g_s=16, F=2, L=2, K_c=4, K_g=8, theta=1e4, hf_wavelength=0.0)
    d.update(kw)
    return oracle.Params(**d)


@pytest.mark.parametrize("hf", [math.inf, 0.0, 1e-9])
def test_group_of_one_token_is_the_rotated_key(hf):
    # With g_s = 1 every group is one token, whose mean position is its own,
    # so the summary is R_p(k) whatever the high/low split.
    rng = np.random.default_rng(2)
    B, T, H, D = 1, 128, 2, 64
    K = rng.standard_normal((B, T, H, D))
    pos = rng.permutation(5000)[:T].astype(np.int32)[None]
    _, S_g = oracle.build_summaries(K, pos, _params(g_s=1, hf_wavelength=hf))
    want = oracle.rope_rows(K[0].transpose(1, 0, 2), np.broadcast_to(pos[0], (H, T)), 1e4)
    np.testing.assert_allclose(S_g[0], want, rtol=0, atol=1e-12)


def test_all_low_identical_keys_rotate_at_mean_position():
    # All pairs low, every key of a chunk the same k: summary = R_{p_mid}(k)
    # with p_mid the mean position (here irregular positions).
    rng = np.random.default_rng(3)
    D = 64
    k = rng.standard_normal(D)
    K = np.broadcast_to(k, (1, 64, 1, D)).copy()
    pos = np.sort(rng.choice(10000, 64, replace=False)).astype(np.int32)[None]
    S_c, S_g = oracle.build_summaries(K, pos, _params(hf_wavelength=1e-9))
    np.testing.assert_allclose(S_c[0, 0, 0], _complex_rotate(k, pos.mean(), 1e4), atol=1e-12)
    for g in range(4):
        pm = pos[0, 16 * g:16 * g + 16].mean()
        np.testing.assert_allclose(S_g[0, 0, g], _complex_rotate(k, pm, 1e4), atol=1e-12)


def test_contiguous_chunk_mid_position_is_start_plus_31_5():
    D = 64
    k = np.random.default_rng(4).standard_normal(D)
    K = np.broadcast_to(k, (1, 192, 1, D)).copy()
    pos = np.arange(192, dtype=np.int32)[None]
    S_c, _ = oracle.build_summaries(K, pos, _params(hf_wavelength=1e-9))
    for m in range(3):
        np.testing.assert_allclose(S_c[0, 0, m], _complex_rotate(k, 64 * m + 31.5, 1e4),
                                   atol=1e-12)


def test_all_high_summary_is_mean_of_rotated_keys_and_of_groups():
    rng = np.random.default_rng(5)
    B, T, H, D = 2, 256, 3, 32
    K = rng.standard_normal((B, T, H, D))
    pos = (np.arange(T)[None] + np.array([[0], [777]])).astype(np.int32)
    S_c, S_g = oracle.build_summaries(K, pos, _params(hf_wavelength=math.inf))
    for b in range(B):
        for h in range(H):
            rot = _complex_rotate(K[b, :, h], pos[b].astype(np.float64), 1e4)
            np.testing.assert_allclose(S_c[b, h], rot.reshape(4, 64, D).mean(1), atol=1e-12)
            np.testing.assert_allclose(S_g[b, h], rot.reshape(16, 16, D).mean(1), atol=1e-12)
            np.testing.assert_allclose(S_c[b, h], S_g[b, h].reshape(4, 4, D).mean(1), atol=1e-12)


def test_mixed_summary_splits_pairs():
    # Each pair of the mixed summary equals the all-high summary on high
    # pairs and the all-low summary on low pairs.
    rng = np.random.default_rng(6)
    K = rng.standard_normal((1, 128, 1, 64))
    pos = np.arange(128, dtype=np.int32)[None] + 3000
    mix = oracle.build_summaries(K, pos, _params())
    hi_all = oracle.build_summaries(K, pos, _params(hf_wavelength=math.inf))
    lo_all = oracle.build_summaries(K, pos, _params(hf_wavelength=1e-9))
    high = oracle.pair_is_high(64, 1e4)
    sel = np.concatenate([high, high])
    for a, h_, l_ in zip(mix, hi_all, lo_all):
        np.testing.assert_array_equal(a[..., sel], h_[..., sel])
        np.testing.assert_array_equal(a[..., ~sel], l_[..., ~sel])
    # and the low part really differs from the per-token rotation
    assert np.abs(hi_all[0][..., ~sel] - lo_all[0][..., ~sel]).max() > 1e-3


def test_open_chunk_has_no_summary():
    K = np.random.default_rng(7).standard_normal((1, 64 * 3 + 17, 1, 64))
    pos = np.arange(K.shape[1], dtype=np.int32)[None]
    S_c, S_g = oracle.build_summaries(K, pos, _params())
    assert S_c.shape[2] == 3 and S_g.shape[2] == 12


def test_scores_are_shift_invariant():
    # Adding the same offset to every position leaves every chunk and group
    # score unchanged: the query and summary rotations use one convention
    # (high pairs: relative angles; low pairs: R_p q . R_{p_mid} k_bar).
    rng = np.random.default_rng(8)
    B, T, Hq, Hkv, D = 1, 640, 4, 2, 64
    Q = rng.standard_normal((B, T, Hq, D))
    K = rng.standard_normal((B, T, Hkv, D))
    V = rng.standard_normal((B, T, Hkv, D))
    p = _params(L=1, K_c=3, K_g=5)
    pos = np.arange(T, dtype=np.int32)[None]
    a = oracle.hga(Q, K, V, pos, p, want_scores=True)
    b = oracle.hga(Q, K, V, pos + 40000, p, want_scores=True)
    for key in ("cscore", "gscore"):
        x, y = a[key], b[key]
        assert np.array_equal(np.isnan(x), np.isnan(y))
        f = ~np.isnan(x)
        assert np.abs(x[f] - y[f]).max() < 1e-8 * max(1.0, np.abs(x[f]).max())
    np.testing.assert_array_equal(a["sel_g"], b["sel_g"])
    np.testing.assert_allclose(a["O"], b["O"], atol=1e-10)
