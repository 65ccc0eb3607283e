"""CPU oracle for HGA routed exact-token attention (fp64, plain C).

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg use it; the CUDA library never imports or calls it.
This wrapper only marshals numpy/torch arrays into the C functions of
``hga_oracle.c`` (built with gcc on first use); every step of the arithmetic
is in that file, with the passage of the method page it follows.

Pinned by the CPU tests (``tests/test_oracle_*.py``): RoPE against complex
rotation and its relative-position property; the high/low pair split against
its closed form; summaries against the g_s=1 and identical-key special cases
and linearity; top-K against brute-force enumeration; the visible set against
the policy's invariants; full-budget HGA against dense eq. (1); dense eq. (1)
against a library softmax attention; the backward against automatic
differentiation of dense attention (full budget), central differences of the
forward (routed sets), its sum rules and position-shift invariance.  Parity unpinned: the readings R1-R3 of
``hga_oracle.c`` (pair convention, high/low threshold, p_mid) beyond those
special cases are readings of the page, not facts it prints.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile hga_oracle.c into liboracle.so (gcc -O2, pthreads)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Params(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int32), ("g_s", ctypes.c_int32), ("F", ctypes.c_int32),
                ("L", ctypes.c_int32), ("K_c", ctypes.c_int32), ("K_g", ctypes.c_int32),
                ("theta", ctypes.c_double), ("hf_wavelength", ctypes.c_double)]


@dataclass(frozen=True)
class Params:
    C: int = 64
    g_s: int = 16
    F: int = 2
    L: int = 2
    K_c: int = 4
    K_g: int = 8
    theta: float = 1e4
    hf_wavelength: float = 0.0   # <= 0: the chunk length C

    @staticmethod
    def of(w, **kw) -> "Params":
        d = dict(C=w.C, g_s=w.g_s, F=w.F, L=w.L, K_c=w.K_c, K_g=w.K_g, theta=w.theta)
        d.update(kw)
        return Params(**d)

    def c(self) -> _Params:
        return _Params(self.C, self.g_s, self.F, self.L, self.K_c, self.K_g,
                       float(self.theta), float(self.hf_wavelength))


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            lib.or_omega.argtypes = [i32, dbl, P]
            lib.or_pair_is_high.argtypes = [i32, dbl, dbl, i32, P]
            lib.or_rope_rows.argtypes = [P, P, i64, i32, dbl, P]
            lib.or_set_summary.argtypes = [P, i64, P, i64, i32, i32, P, P, P]
            lib.or_build_summaries.argtypes = [P, P, i32, i32, i32, i32, P, P, P]
            lib.or_route_query.argtypes = [P, P, i32, i32, i32, i32, dbl, i32, i32, i32, i32, P]
            lib.or_topk.argtypes = [P, P, i32, i32, P]
            lib.or_topk.restype = i32
            lib.or_route.argtypes = [P, P, P, i32, i32, i32, P, P, P, P, P]
            lib.or_visible_mark.argtypes = [i32, i32, i32, P, P, P]
            lib.or_attend_row.argtypes = [P, P, P, i64, P, i32, i32, P, P]
            lib.or_hga.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, i32, P, i32, i32,
                                   P, P, P, P, P, P, P, i32]
            lib.or_hga.restype = i32
            lib.or_dense.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, dbl, P, P]
            lib.or_dense.restype = i32
            lib.or_hga_backward.argtypes = [P, P, P, P, P, i32, i32, i32, i32, i32, P, P, i32,
                                            P, P, P]
            lib.or_hga_backward.restype = i32
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening to a contiguous float64 array (torch or numpy input)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def omega(D: int, theta: float) -> np.ndarray:
    out = np.empty(D // 2, np.float64)
    _load().or_omega(D, theta, _p(out))
    return out


def pair_is_high(D: int, theta: float, hf_wavelength: float = 0.0, C: int = 64) -> np.ndarray:
    out = np.empty(D // 2, np.int32)
    _load().or_pair_is_high(D, theta, hf_wavelength, C, _p(out))
    return out.astype(bool)


def rope_rows(x, pos, theta: float) -> np.ndarray:
    x = _f64(x)
    D = x.shape[-1]
    xf = x.reshape(-1, D)
    pf = _f64(pos).reshape(-1)
    assert pf.shape[0] == xf.shape[0]
    out = np.empty_like(xf)
    _load().or_rope_rows(_p(xf), _p(pf), xf.shape[0], D, theta, _p(out))
    return out.reshape(x.shape)


def set_summary(k_rows, pos, theta: float, hf_wavelength: float = 0.0, C: int = 64) -> np.ndarray:
    """Mixed-RoPE summary of one token set (rows [n, D], positions [n])."""
    k = _f64(k_rows)
    n, D = k.shape
    pos = _i32(pos).reshape(-1)
    om = omega(D, theta)
    hi = pair_is_high(D, theta, hf_wavelength, C).astype(np.int32)
    out = np.empty(D, np.float64)
    _load().or_set_summary(_p(k), D, _p(pos), 0, n, D, _p(om), _p(hi), _p(out))
    return out


def build_summaries(K, pos, params: Params):
    """K [B,T,Hkv,D] -> S_c [B,Hkv,NC,D], S_g [B,Hkv,NG,D] (fp64)."""
    K = _f64(K)
    B, T, Hkv, D = K.shape
    pos = _i32(pos)
    NC = T // params.C
    NG = NC * (params.C // params.g_s)
    S_c = np.zeros((B, Hkv, NC, D), np.float64)
    S_g = np.zeros((B, Hkv, NG, D), np.float64)
    pc = params.c()
    _load().or_build_summaries(_p(K), _p(pos), B, T, Hkv, D, ctypes.byref(pc), _p(S_c), _p(S_g))
    return S_c, S_g


def route_query(Q, pos, Hkv: int, theta: float, b: int, h: int, i0: int, i1: int) -> np.ndarray:
    Q = _f64(Q)
    B, T, Hq, D = Q.shape
    pos = _i32(pos)
    out = np.empty(D, np.float64)
    _load().or_route_query(_p(Q), _p(pos), T, Hq, Hkv, D, theta, b, h, i0, i1, _p(out))
    return out


def topk(scores, ids, K: int):
    s = _f64(scores).reshape(-1)
    i = _i32(ids).reshape(-1)
    out = np.empty(max(K, 1), np.int32)
    kept = _load().or_topk(_p(s), _p(i), s.shape[0], K, _p(out))
    return out[:K], kept


def route(q_r, S_c_bh, S_g_bh, c: int, params: Params):
    """Two-level routing for one (batch, KV head) and current chunk c."""
    q_r = _f64(q_r)
    S_c_bh = _f64(S_c_bh)
    S_g_bh = _f64(S_g_bh)
    NC, D = S_c_bh.shape
    NG = S_g_bh.shape[0]
    sel_c = np.empty(max(params.K_c, 1), np.int32)
    sel_g = np.empty(max(params.K_g, 1), np.int32)
    cs = np.empty(max(NC, 1), np.float64)
    gs = np.empty(max(NG, 1), np.float64)
    pc = params.c()
    _load().or_route(_p(q_r), _p(S_c_bh), _p(S_g_bh), NC, c, D, ctypes.byref(pc),
                     _p(sel_c), _p(sel_g), _p(cs), _p(gs))
    return sel_c[:params.K_c], sel_g[:params.K_g], cs[:NC], gs[:NG]


def visible_mark(c: int, i: int, T: int, sel_g, params: Params) -> np.ndarray:
    sg = _i32(sel_g).reshape(-1)
    if sg.shape[0] < params.K_g:
        sg = np.concatenate([sg, -np.ones(params.K_g - sg.shape[0], np.int32)])
    mark = np.zeros(max(T, 1), np.uint8)
    pc = params.c()
    _load().or_visible_mark(c, i, T, _p(sg), ctypes.byref(pc), _p(mark))
    return mark[:T].astype(bool)


def hga(Q, K, V, pos, params: Params, route_block: int | None = None, units=None,
        nthreads: int | None = None, want_scores: bool = False, sel_g_force=None,
        attend: bool = True):
    """Full HGA over query sets.  route_block = C (prefill blocks, default) or
    1 (per-token routing, as in decode).  units: list of (b, s) pairs; default
    every query set of every batch row.  Returns dict with O [B,T,Hq,D] (rows
    of the computed units; NaN elsewhere), LSE [B,Hq,T], units, sel_c
    [n_units,Hkv,K_c], sel_g [n_units,Hkv,K_g] and optionally cscore/gscore.
    sel_g_force [n_units,Hkv,K_g]: attend over these routed groups instead of
    the oracle's own choice.  attend=False: routing only."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    pos = _i32(pos)
    B, T, Hq, D = Q.shape
    Hkv = K.shape[2]
    rb = params.C if route_block is None else int(route_block)
    nsets = (T + rb - 1) // rb
    if units is None:
        units = [(b, s) for b in range(B) for s in range(nsets)]
    u = np.ascontiguousarray(np.asarray(units, dtype=np.int32).reshape(-1, 2))
    nu = u.shape[0]
    NC = T // params.C
    NG = NC * (params.C // params.g_s)
    O = np.full((B, T, Hq, D), np.nan, np.float64)
    LSE = np.full((B, Hq, T), np.nan, np.float64)
    sel_c = np.full((nu, Hkv, max(params.K_c, 1)), -2, np.int32)
    sel_g = np.full((nu, Hkv, max(params.K_g, 1)), -2, np.int32)
    cs = np.full((nu, Hkv, max(NC, 1)), np.nan) if want_scores else None
    gs = np.full((nu, Hkv, max(NG, 1)), np.nan) if want_scores else None
    if nthreads is None:
        nthreads = len(os.sched_getaffinity(0))
    force = None
    if sel_g_force is not None:
        force = np.ascontiguousarray(_i32(sel_g_force).reshape(nu, Hkv, params.K_g))
    pc = params.c()
    rc = _load().or_hga(_p(Q), _p(K), _p(V), _p(pos), B, T, Hq, Hkv, D, ctypes.byref(pc), rb,
                        _p(u), nu, int(nthreads), _p(O), _p(LSE), _p(sel_c), _p(sel_g),
                        _p(cs) if want_scores else None, _p(gs) if want_scores else None,
                        _p(force) if force is not None else None, 1 if attend else 0)
    if rc != 0:
        raise ValueError("oracle: malformed arguments")
    out = {"O": O, "LSE": LSE, "units": u, "sel_c": sel_c[:, :, :params.K_c],
           "sel_g": sel_g[:, :, :params.K_g], "nthreads": int(nthreads)}
    if want_scores:
        out["cscore"] = cs[:, :, :NC]
        out["gscore"] = gs[:, :, :NG]
    return out


def dense(Q, K, V, pos, theta: float):
    """Dense causal attention, eq. (1): O [B,T,Hq,D], LSE [B,Hq,T]."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    pos = _i32(pos)
    B, T, Hq, D = Q.shape
    Hkv = K.shape[2]
    O = np.empty((B, T, Hq, D), np.float64)
    LSE = np.empty((B, Hq, T), np.float64)
    rc = _load().or_dense(_p(Q), _p(K), _p(V), _p(pos), B, T, Hq, Hkv, D, theta, _p(O), _p(LSE))
    if rc != 0:
        raise ValueError("oracle: malformed arguments")
    return O, LSE


def hga_backward(Q, K, V, pos, dO, params: Params, sel_g, nthreads: int | None = None):
    """Gradients of the HGA prefill attention with the routed groups held
    fixed: sel_g [B, NB, Hkv, K_g] are the groups the forward attended (the
    routing is a discrete choice).  dO [B,T,Hq,D] is the gradient of the loss
    with respect to O.  Returns (dQ, dK, dV) with respect to the raw
    (pre-RoPE) q and k, and v, as fp64 arrays."""
    Q = _f64(Q)
    K = _f64(K)
    V = _f64(V)
    dO = _f64(dO)
    pos = _i32(pos)
    B, T, Hq, D = Q.shape
    Hkv = K.shape[2]
    NB = (T + params.C - 1) // params.C
    sg = np.ascontiguousarray(_i32(sel_g).reshape(B, NB, Hkv, params.K_g))
    dQ = np.empty_like(Q)
    dK = np.empty_like(K)
    dV = np.empty_like(V)
    if nthreads is None:
        nthreads = len(os.sched_getaffinity(0))
    pc = params.c()
    rc = _load().or_hga_backward(_p(Q), _p(K), _p(V), _p(pos), _p(dO), B, T, Hq, Hkv, D,
                                 ctypes.byref(pc), _p(sg), int(nthreads), _p(dQ), _p(dK), _p(dV))
    if rc != 0:
        raise ValueError("oracle: malformed arguments")
    return dQ, dK, dV
