"""Comparison rules between the CUDA path and the CPU oracle.

* Routed index sets must be identical, except where the oracle's own scores
  tie at the selection boundary: two candidates tie when their fp64 scores
  differ by at most 1e-6 of the dot product's magnitude scale sum_d |q_d s_d|
  (the method fixes no precision; the GPU ranks fp32-rounded scores of fp64
  dot products of fp32 summaries).  When the chunk sets differ by a tie, the
  group set is checked against the oracle's top-K over the GPU's chunks.
* Outputs: per (token, head) row, max|o_gpu - o_ref| / max|o_ref| must stay
  within 1e-5 for fp32 inputs and 2e-2 for bf16 inputs (fp32 accumulation).
  Rows whose routed set differs by a tie are compared with an oracle run that
  attends over the GPU's routed set.
"""
from __future__ import annotations

import numpy as np

import oracle

TIE_REL = 1e-6
TOL = {"f32": 1e-5, "bf16": 2e-2}


def row_rel_err(gpu, ref):
    """max over rows of max|gpu - ref| / max|ref| (last axis = the row)."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    num = np.abs(g - r).max(-1)
    den = np.abs(r).max(-1)
    den = np.where(den == 0, 1.0, den)
    return float((num / den).max()) if num.size else 0.0


class RouteRef:
    """Oracle quantities needed to judge one (unit, KV head) selection."""

    def __init__(self, Q, K, pos, p: oracle.Params, Hkv: int):
        self.Q = Q
        self.pos = pos
        self.p = p
        self.Hkv = Hkv
        self.S_c, self.S_g = oracle.build_summaries(K, pos, p)

    def q_r(self, b, h, i0, i1):
        return oracle.route_query(self.Q, self.pos, self.Hkv, self.p.theta, b, h, i0, i1)


def _tie_ok(gset, oset, score, scale):
    if gset == oset:
        return True
    if len(gset) != len(oset):
        return False
    if not oset:
        return True
    kth = min(oset, key=lambda i: score[i])
    for i in gset ^ oset:
        tol = TIE_REL * max(scale[i], scale[kth])
        if abs(score[i] - score[kth]) > tol:
            return False
    return True


def check_unit_selection(ref: RouteRef, b, h, i0, i1, c, gpu_c, gpu_g, orc_c, orc_g):
    """Returns (ok, tie_differs) for one unit and KV head."""
    p = ref.p
    q = ref.q_r(b, h, i0, i1)
    Sc = ref.S_c[b, h]
    Sg = ref.S_g[b, h]
    cs, ca = Sc @ q, np.abs(Sc) @ np.abs(q)
    gs, ga = Sg @ q, np.abs(Sg) @ np.abs(q)
    G = set(int(x) for x in gpu_c if x >= 0)
    O = set(int(x) for x in orc_c if x >= 0)
    if not _tie_ok(G, O, cs, ca):
        return False, True
    # groups: oracle's top-K_g over the groups of the GPU's chunks
    cand = np.array([m * (p.C // p.g_s) + g for m in sorted(G) for g in range(p.C // p.g_s)],
                    np.int32)
    if G == O:
        want = set(int(x) for x in orc_g if x >= 0)
    else:
        sel, kept = oracle.topk(gs[cand], cand, p.K_g) if cand.size else (np.zeros(0), 0)
        want = set(int(x) for x in sel[:kept])
    got = set(int(x) for x in gpu_g if x >= 0)
    if not _tie_ok(got, want, gs, ga):
        return False, True
    # padding and ordering
    for arr, k in ((gpu_c, p.K_c), (gpu_g, p.K_g)):
        a = np.asarray(arr)
        n = int((a >= 0).sum())
        if not (np.all(a[:n] >= 0) and np.all(a[n:] == -1) and np.all(np.diff(a[:n]) > 0)):
            return False, False
    return True, (got != set(int(x) for x in orc_g if x >= 0))
