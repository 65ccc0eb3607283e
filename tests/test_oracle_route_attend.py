"""Pins of the oracle's routing, visible set and attention.

Method page: HGA paper review, section 3: routing policy (deterministic
visibility, middle routing, the two-level selection equation), exact token
output attention, eq. (1); section 6 setup table and Table 4 (1.9% at 64K);
Table 7 (full coverage equals causal SDPA).
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_prefill_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _params(**kw):
    d = dict(C=64, g_s=16, F=2, L=2, K_c=4, K_g=8, theta=1e4, hf_wavelength=0.0)
    d.update(kw)
    return oracle.Params(**d)


def _brute_topk(scores, ids, K):
    """The unique subset S (|S| = min(K, n)) such that every member beats
    every non-member: higher score, or equal score and lower id."""
    n = len(scores)
    k = min(K, n)
    beats = lambda a, b: scores[a] > scores[b] or (scores[a] == scores[b] and ids[a] < ids[b])
    if n > 10:
        # too many subsets to list: a member is beaten by fewer than K others
        return sorted(ids[a] for a in range(n) if sum(beats(b, a) for b in range(n)) < K)
    found = []
    for S in itertools.combinations(range(n), k):
        rest = [j for j in range(n) if j not in S]
        if all(beats(a, b) for a in S for b in rest):
            found.append(sorted(ids[a] for a in S))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("seed", range(40))
def test_topk_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(0, 10))
    K = int(rng.integers(0, 8))
    scores = rng.integers(-3, 4, n).astype(np.float64)   # many exact ties
    ids = rng.permutation(100)[:n].astype(np.int32)
    got, kept = oracle.topk(scores, ids, K)
    want = _brute_topk(list(scores), list(ids), K)
    assert kept == len(want)
    assert list(got[:kept]) == want and (got[kept:] == -1).all()


def _middle(c, F, L):
    return [m for m in range(c) if F <= m <= c - L - 1 and not (L == 0 and m == c - 1)]


@pytest.mark.parametrize("F,L,K_c,K_g", [(2, 2, 4, 8), (0, 0, 3, 5), (1, 3, 2, 8), (2, 8, 16, 32),
                                         (3, 1, 0, 4), (2, 2, 6, 0)])
def test_route_candidates_and_selection(F, L, K_c, K_g):
    rng = np.random.default_rng(F * 100 + L * 10 + K_c)
    NC, D, g_s = 24, 32, 16
    p = _params(F=F, L=L, K_c=K_c, K_g=K_g, g_s=g_s)
    S_c = rng.standard_normal((NC, D))
    S_g = rng.standard_normal((NC * 4, D))
    q_r = rng.standard_normal(D)
    for c in range(NC + 1):
        sel_c, sel_g, cs, gs = oracle.route(q_r, S_c, S_g, c, p)
        mid = _middle(c, F, L)
        assert sorted(np.flatnonzero(~np.isnan(cs))) == mid
        np.testing.assert_allclose(cs[mid], S_c[mid] @ q_r, rtol=1e-13)
        want_c = _brute_topk([float(x) for x in S_c[mid] @ q_r], mid, K_c) if mid else []
        kc = len(want_c)
        assert list(sel_c[:kc]) == want_c and (sel_c[kc:] == -1).all()
        cand = [m * 4 + g for m in want_c for g in range(4)]
        assert sorted(np.flatnonzero(~np.isnan(gs))) == sorted(cand)
        want_g = _brute_topk([float(x) for x in S_g[cand] @ q_r], cand, K_g) if cand else []
        kg = len(want_g)
        assert list(sel_g[:kg]) == want_g and (sel_g[kg:] == -1).all()
        # routed groups never touch the always-visible windows
        assert all(F <= g // 4 <= c - max(L, 1) - 1 for g in want_g)


def test_route_query_sums_rotated_queries_over_block_and_heads():
    rng = np.random.default_rng(11)
    B, T, Hq, Hkv, D = 2, 130, 6, 2, 16
    Q = rng.standard_normal((B, T, Hq, D))
    pos = np.tile(np.arange(T, dtype=np.int32), (B, 1)) + 7
    q_r = oracle.route_query(Q, pos, Hkv, 1e4, 1, 1, 64, 128)
    rows = Q[1, 64:128, 3:6].reshape(-1, D)
    prow = np.repeat(pos[1, 64:128], 3).astype(np.float64)
    want = oracle.rope_rows(rows, prow, 1e4).sum(0)
    np.testing.assert_allclose(q_r, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("F,L", [(2, 2), (0, 0), (3, 0), (1, 5)])
def test_visible_set_policy(F, L):
    p = _params(F=F, L=L, K_g=3)
    C = 64
    T = 20 * C
    sel_g = np.array([4 * 9 + 1, 4 * 12, -1], np.int32)
    for c in [0, 1, 3, 13, 19]:
        for i in [c * C, c * C + 17, c * C + 63]:
            mk = oracle.visible_mark(c, i, T, sel_g if c >= 14 else np.full(3, -1), p)
            assert not mk[i + 1:].any()                           # causal
            assert mk[c * C:i + 1].all()                          # current chunk up to i
            for m in range(min(F, c)):
                assert mk[m * C:(m + 1) * C].all()                # sinks
            for m in range(max(0, c - L), c):
                assert mk[m * C:(m + 1) * C].all()                # recent
            if c >= 1:
                assert mk[(c - 1) * C:c * C].all()                # forced previous chunk
            if c >= 14:
                assert mk[(4 * 9 + 1) * 16:(4 * 9 + 2) * 16].all()
                assert mk[(4 * 12) * 16:(4 * 12 + 1) * 16].all()
            fixed = set(range(min(F, c))) | set(range(max(0, c - L), c)) | ({c - 1} if c else set())
            n_routed = 2 * 16 if c >= 14 else 0
            assert mk.sum() == len(fixed) * C + (i - c * C + 1) + n_routed


def _golden():
    d = {}
    for line in open(os.path.join(GOLDEN, "pages_setup.txt")):
        line = line.split("#")[0].strip()
        if line:
            k, v = (s.strip() for s in line.split("="))
            d[k] = float(v)
    return d


def test_visible_budget_matches_pages_sparsity_at_64k():
    # Setup table: C=64, 2 sink chunks, 8 recent chunks; Table 4: about 1.9%
    # of a 64K context is attended.  With K_g=32 groups of 16 the visible set
    # at a block end is 128 + 512 + 64 + 512 = 1216 tokens = 1.86%.
    g = _golden()
    C = int(g["chunk_size"])
    F = int(g["sink_tokens"]) // C
    L = int(g["recent_tokens"]) // C
    T = int(g["niah_context"])
    p = _params(C=C, F=F, L=L, K_c=int(g["routed_chunks"]), K_g=32, g_s=int(g["group_size_smalllm"]))
    c = T // C - 1
    sel_g = np.arange(32, dtype=np.int32) * 4 + 40
    mk = oracle.visible_mark(c, T - 1, T, sel_g, p)
    assert mk.sum() == 1216
    assert round(100.0 * mk.sum() / T, 1) == g["niah_sparsity_pct"]


def _sdpa_f64(Q, K, V, pos, theta, mask=None):
    """torch's scaled_dot_product_attention in fp64 on RoPE'd q and k."""
    B, T, Hq, D = Q.shape
    Hkv = K.shape[2]
    qr = oracle.rope_rows(Q, np.broadcast_to(pos[:, :, None], (B, T, Hq)), theta)
    kr = oracle.rope_rows(K, np.broadcast_to(pos[:, :, None], (B, T, Hkv)), theta)
    q = torch.from_numpy(qr).permute(0, 2, 1, 3)
    k = torch.from_numpy(kr).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    v = torch.from_numpy(np.asarray(V, np.float64)).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    if mask is None:
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=torch.from_numpy(mask))
    return o.permute(0, 2, 1, 3).numpy()


def test_dense_eq1_matches_library_sdpa():
    rng = np.random.default_rng(12)
    B, T, Hq, Hkv, D = 2, 150, 4, 2, 32
    Q, K, V = rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    pos = np.tile(np.arange(T, dtype=np.int32), (B, 1))
    O, LSE = oracle.dense(Q, K, V, pos, 1e4)
    np.testing.assert_allclose(O, _sdpa_f64(Q, K, V, pos, 1e4), atol=1e-12)
    # LSE: log of the softmax denominator, checked by brute force on one row
    qr = oracle.rope_rows(Q[1, 99, 3], [99], 1e4)
    kr = oracle.rope_rows(K[1, :100, 1], np.arange(100.0), 1e4)
    s = kr @ qr / math.sqrt(D)
    assert abs(LSE[1, 3, 99] - (s.max() + math.log(np.exp(s - s.max()).sum()))) < 1e-12


@pytest.mark.parametrize("T,F,L,g_s,Hq,Hkv", [(1024, 2, 2, 16, 2, 1), (700, 1, 0, 8, 4, 2),
                                              (64 * 5 + 9, 0, 3, 64, 3, 3), (40, 2, 2, 16, 2, 1)])
def test_full_budget_equals_dense(T, F, L, g_s, Hq, Hkv):
    # A routing budget covering every middle chunk and group opens every
    # token, so routed attention is dense causal attention (Table 7, rows 1-2).
    rng = np.random.default_rng(T)
    B, D = 1, 32
    Q, K, V = rng.standard_normal((B, T, Hq, D)), rng.standard_normal((B, T, Hkv, D)), rng.standard_normal((B, T, Hkv, D))
    pos = np.arange(T, dtype=np.int32)[None]
    nc = T // 64 + 1
    p = _params(F=F, L=L, g_s=g_s, K_c=nc, K_g=nc * (64 // g_s))
    r = oracle.hga(Q, K, V, pos, p)
    want = _sdpa_f64(Q, K, V, pos, 1e4)
    np.testing.assert_allclose(r["O"], want, atol=1e-11)
    r1 = oracle.hga(Q, K, V, pos, p, route_block=1)      # per-token routing too
    np.testing.assert_allclose(r1["O"], want, atol=1e-11)


def test_routed_attention_equals_masked_library_attention():
    # Given the visible sets, the output is softmax attention under that mask.
    w = WORKLOADS["tiny_f32_prefill_1k"]
    q, k, v, pos, _ = make_prefill_inputs(w, seed=3)
    p = oracle.Params.of(w)
    r = oracle.hga(q, k, v, pos, p)
    T = w.T
    mask = np.zeros((1, w.Hq, T, T), bool)
    for u in range(T // 64):
        for i in range(64 * u, 64 * u + 64):
            mask[0, :, i] = oracle.visible_mark(u, i, T, r["sel_g"][u, 0], p)
    want = _sdpa_f64(q.numpy(), k.numpy(), v.numpy(), pos.numpy(), w.theta, mask)
    np.testing.assert_allclose(r["O"], want, atol=1e-11)
    assert not np.allclose(r["O"], oracle.dense(q, k, v, pos, w.theta)[0], atol=1e-3)


def test_degenerate_cases():
    rng = np.random.default_rng(13)
    D = 16
    for T in (1, 5, 64, 65):
        Q, K, V = rng.standard_normal((1, T, 2, D)), rng.standard_normal((1, T, 1, D)), rng.standard_normal((1, T, 1, D))
        pos = np.arange(T, dtype=np.int32)[None]
        r = oracle.hga(Q, K, V, pos, _params())
        np.testing.assert_allclose(r["O"], _sdpa_f64(Q, K, V, pos, 1e4), atol=1e-12)
        assert (r["sel_c"] == -1).all() and (r["sel_g"] == -1).all()
    # first token attends only to itself
    np.testing.assert_allclose(r["O"][0, 0, 0], V[0, 0, 0], atol=1e-14)
    # K_c = 0: only the fixed windows
    T = 640
    Q, K, V = rng.standard_normal((1, T, 2, D)), rng.standard_normal((1, T, 1, D)), rng.standard_normal((1, T, 1, D))
    pos = np.arange(T, dtype=np.int32)[None]
    r = oracle.hga(Q, K, V, pos, _params(K_c=0))
    assert (r["sel_c"] == -1).all() and (r["sel_g"] == -1).all()


def test_planted_topic_chunk_is_routed():
    # Statistical check of the generator + routing: the chunk whose topic the
    # block's queries lean towards wins the chunk top-K almost always.
    w = WORKLOADS["qwen3_30b_a3b_bf16_prefill_32k"].replace(T=4096, B=1)
    q, k, v, pos, info = make_prefill_inputs(w, seed=5)
    p = oracle.Params.of(w)
    units = [(0, b) for b in range(20, 64, 4)]
    r = oracle.hga(q, k, v, pos, p, units=units)
    hits = sum(int(info["planted"][0, b]) in r["sel_c"][i, h]
               for i, (_, b) in enumerate(units) for h in range(w.Hkv))
    assert hits >= 0.9 * len(units) * w.Hkv
