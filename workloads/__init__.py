"""Seeded synthetic inputs for routed exact-token attention (HGA).

This module only draws input data.  It holds none of the method's arithmetic:
no RoPE, no summaries, no routing, no attention.  Both the CPU oracle (through
the tests and the bench) and the CUDA library receive exactly the arrays built
here, so the two sides never share code, only data.

Recipes (one per workload; every draw is from ``torch.Generator`` seeded with
``seed``, on the CPU for small cases or on a CUDA device for the large ones):

* ``iid``      Q, K, V i.i.d. N(0, 1).
* ``topic``    K[b, t, h] = topic[b, h, t // C] + sigma * N(0, I); the chunk
               topic vectors are N(0, I).  Q and V are N(0, 1).
* ``planted``  K as in ``topic``.  Each query block (64 tokens) of batch row b
               picks one earlier *middle* chunk m* uniformly; every query row
               (token, head) of that block is z ~ N(0, I) bent so that its
               cosine with the topic of m* (for the head's KV head) is 0.5:
               q = |z| (0.5 t_hat + sqrt(0.75) u_hat), u_hat the unit part of z
               orthogonal to t_hat.  Blocks without a middle chunk keep q = z.
               V is N(0, 1).

Values for bf16 workloads are drawn in fp32 and rounded to bf16 (round to
nearest even, by ``torch.Tensor.to``); the oracle widens those bf16 values
exactly.  Positions are ``arange(T)`` per batch row (int32).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = ["Workload", "WORKLOADS", "make_prefill_inputs", "make_decode_inputs",
           "middle_range"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    Hq: int
    Hkv: int
    D: int
    theta: float
    C: int = 64
    g_s: int = 16
    F: int = 2
    L: int = 2
    K_c: int = 4
    K_g: int = 8
    dtype: str = "f32"          # "f32" or "bf16"
    recipe: str = "iid"         # "iid" | "topic" | "planted"
    sigma: float = 0.5
    steps: int = 0              # decode steps appended after the T-token cache

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads of the hot path, named by what they are.
WORKLOADS = {
    "tiny_f32_prefill_1k": Workload(
        "tiny_f32_prefill_1k", B=1, T=1024, Hq=2, Hkv=1, D=64, theta=1e4,
        g_s=16, F=2, L=2, K_c=4, K_g=8, dtype="f32", recipe="iid"),
    "smalllm40m_bf16_prefill_4k": Workload(
        "smalllm40m_bf16_prefill_4k", B=8, T=4096, Hq=8, Hkv=8, D=64, theta=1e4,
        g_s=16, F=2, L=8, K_c=8, K_g=16, dtype="bf16", recipe="topic"),
    "qwen3_30b_a3b_bf16_prefill_32k": Workload(
        "qwen3_30b_a3b_bf16_prefill_32k", B=1, T=32768, Hq=32, Hkv=4, D=128,
        theta=1e6, g_s=16, F=2, L=8, K_c=16, K_g=32, dtype="bf16",
        recipe="planted"),
    "qwen3_30b_a3b_bf16_decode_64k": Workload(
        "qwen3_30b_a3b_bf16_decode_64k", B=16, T=65536, Hq=32, Hkv=4, D=128,
        theta=1e6, g_s=16, F=2, L=8, K_c=16, K_g=32, dtype="bf16",
        recipe="planted", steps=256),
    "qwen3_30b_a3b_bf16_hosttier_prefill_64k": Workload(
        "qwen3_30b_a3b_bf16_hosttier_prefill_64k", B=1, T=65536, Hq=32, Hkv=4,
        D=128, theta=1e6, g_s=16, F=2, L=8, K_c=16, K_g=32, dtype="bf16",
        recipe="planted"),
}


def middle_range(c: int, F: int, L: int):
    """Chunk indices a query in chunk ``c`` may route to (the generator needs
    only the range to plant a topic; it is the same rule the method states:
    closed chunks after the F sinks and before the L recent ones, with the
    forced previous chunk removed when L == 0)."""
    hi = c - L - 1
    if L == 0:
        hi = c - 2
    return F, hi


def _torch_dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, device):
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32)


def _keys(w: Workload, g, T: int, device) -> torch.Tensor:
    if w.recipe == "iid":
        return _randn(g, (w.B, T, w.Hkv, w.D), device)
    nchunks = (T + w.C - 1) // w.C
    topic = _randn(g, (w.B, nchunks, w.Hkv, w.D), device)
    noise = _randn(g, (w.B, T, w.Hkv, w.D), device)
    k = topic.repeat_interleave(w.C, dim=1)[:, :T] + w.sigma * noise
    return k, topic


def _bend(z: torch.Tensor, t: torch.Tensor) -> torch.Tensor:
    """Rows z (..., D) bent to cosine 0.5 with the matching rows of t."""
    that = t / t.norm(dim=-1, keepdim=True)
    par = (z * that).sum(-1, keepdim=True)
    u = z - par * that
    uhat = u / u.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    return z.norm(dim=-1, keepdim=True) * (0.5 * that + math.sqrt(0.75) * uhat)


def make_prefill_inputs(w: Workload, seed: int = 0, device="cpu", T: Optional[int] = None):
    """Q [B,T,Hq,D], K [B,T,Hkv,D], V [B,T,Hkv,D] (workload dtype) and
    pos [B,T] int32, plus ``info`` (planted chunk per block, or None)."""
    T = w.T if T is None else T
    g = _gen(seed, device)
    info = {"planted": None}
    if w.recipe == "iid":
        k = _keys(w, g, T, device)
        topic = None
    else:
        k, topic = _keys(w, g, T, device)
    q = _randn(g, (w.B, T, w.Hq, w.D), device)
    v = _randn(g, (w.B, T, w.Hkv, w.D), device)
    if w.recipe == "planted":
        nb = (T + w.C - 1) // w.C
        planted = torch.full((w.B, nb), -1, dtype=torch.int64)
        u = torch.rand(w.B, nb, generator=g, device=device).cpu()
        for b in range(w.B):
            for blk in range(nb):
                lo, hi = middle_range(blk, w.F, w.L)
                if hi >= lo:
                    planted[b, blk] = lo + min(int(u[b, blk] * (hi - lo + 1)), hi - lo)
        # topic rows for every (b, token, q-head)
        pl = planted.to(device)
        has = pl >= 0
        pidx = pl.clamp_min(0)                                   # [B, nb]
        tok_blk = torch.arange(T, device=device) // w.C          # [T]
        m_tok = pidx[:, tok_blk]                                 # [B, T]
        has_tok = has[:, tok_blk]                                # [B, T]
        kvh = torch.arange(w.Hq, device=device) // w.G           # [Hq]
        bidx = torch.arange(w.B, device=device)[:, None, None]
        trow = topic[bidx, m_tok[:, :, None], kvh[None, None, :]]  # [B,T,Hq,D]
        bent = _bend(q, trow)
        q = torch.where(has_tok[:, :, None, None], bent, q)
        info["planted"] = planted
    dt = _torch_dtype(w)
    pos = torch.arange(T, dtype=torch.int32, device=device).repeat(w.B, 1)
    return (q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(),
            pos.contiguous(), info)


def make_decode_inputs(w: Workload, seed: int = 0, device="cpu", T: Optional[int] = None,
                       steps: Optional[int] = None):
    """A T-token history (K, V, pos) per sequence and ``steps`` new tokens.

    Returns dict with k_hist, v_hist [B,T,Hkv,D], pos_hist [B,T], and per step
    q [S,B,Hq,D], k_new/v_new [S,B,Hkv,D], pos_new [S,B] (workload dtype /
    int32).  The full sequence (history + new tokens) is drawn exactly as a
    prefill of T + S tokens would be, so token t's key follows its chunk topic;
    step s's query is planted on a random middle chunk of its own chunk."""
    T = w.T if T is None else T
    S = w.steps if steps is None else steps
    Ttot = T + S
    g = _gen(seed, device)
    if w.recipe == "iid":
        k = _keys(w, g, Ttot, device)
        topic = None
    else:
        k, topic = _keys(w, g, Ttot, device)
    v = _randn(g, (w.B, Ttot, w.Hkv, w.D), device)
    q = _randn(g, (S, w.B, w.Hq, w.D), device)
    planted = None
    if w.recipe == "planted" and S > 0:
        u = torch.rand(S, w.B, generator=g, device=device).cpu()
        planted = torch.full((S, w.B), -1, dtype=torch.int64)
        for s in range(S):
            c = (T + s) // w.C
            lo, hi = middle_range(c, w.F, w.L)
            if hi >= lo:
                for b in range(w.B):
                    planted[s, b] = lo + min(int(u[s, b] * (hi - lo + 1)), hi - lo)
        kvh = torch.arange(w.Hq, device=device) // w.G
        pl = planted.to(device)
        bidx = torch.arange(w.B, device=device)[None, :, None]
        trow = topic[bidx, pl.clamp_min(0)[:, :, None], kvh[None, None, :]]  # [S,B,Hq,D]
        q = torch.where((pl >= 0)[:, :, None, None], _bend(q, trow), q)
    dt = _torch_dtype(w)
    pos = torch.arange(Ttot, dtype=torch.int32, device=device).repeat(w.B, 1)
    k = k.to(dt)
    v = v.to(dt)
    return {
        "k_hist": k[:, :T].contiguous(), "v_hist": v[:, :T].contiguous(),
        "pos_hist": pos[:, :T].contiguous(),
        "q": q.to(dt).contiguous(),
        "k_new": k[:, T:].transpose(0, 1).contiguous(),
        "v_new": v[:, T:].transpose(0, 1).contiguous(),
        "pos_new": pos[:, T:].transpose(0, 1).contiguous(),
        "planted": planted,
    }
