"""Python binding of libhga.so, the sm_100a library for HGA routed
exact-token attention (the C ABI is include/hga.h).

This module only marshals torch tensors into the C calls: it checks device,
dtype, shape and contiguity, passes data pointers, sizes and the current
CUDA stream, and raises on a non-OK status.  Every step of the computation
runs in the library's CUDA kernels; there is no CPU fallback, and every call
fails loudly if the library is missing or no CUDA device is present.

Function names follow the C ABI: hga_build_summaries, hga_route, hga_attend,
hga_forward (prefill and decode), hga_workspace_size.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading
from typing import Optional

import torch

__all__ = ["HGAParams", "KVCache", "load", "lib_path", "hga_build_summaries", "hga_route",
           "hga_attend", "hga_forward", "hga_forward_prefill", "hga_forward_decode",
           "hga_workspace_size", "hga_forward_prefill_noalloc", "hga_fill_cache",
           "decode_workspace", "hga_forward_prefill_hostkv", "HGAError", "PREFILL",
           "DECODE", "PREFILL_HOSTKV", "ATTEND_BACKWARD", "hga_device_status",
           "hga_hostkv_link_bytes", "hga_attend_backward", "hga_hostkv_plan",
           "hostkv_workspace_bytes"]

PREFILL, DECODE, PREFILL_HOSTKV, ATTEND_BACKWARD = 0, 1, 2, 3
_F32, _BF16 = 0, 1
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libhga.so")
_lib = None
_lock = threading.Lock()


class HGAError(RuntimeError):
    pass


# ------------------------------------------------------------ C structs --

class _Params(ctypes.Structure):
    _fields_ = [("C", ctypes.c_int32), ("g_s", ctypes.c_int32), ("F", ctypes.c_int32),
                ("L", ctypes.c_int32), ("K_c", ctypes.c_int32), ("K_g", ctypes.c_int32),
                ("rope_theta", ctypes.c_double), ("hf_wavelength", ctypes.c_double)]


class _Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class _Cache(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int32), ("k_rot", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("pos", ctypes.c_void_p), ("k_open", ctypes.c_void_p),
                ("s_chunk", ctypes.c_void_p), ("s_group", ctypes.c_void_p),
                ("lens", ctypes.c_void_p)]


class _HostkvPlan(ctypes.Structure):
    _fields_ = [("wave_blocks", ctypes.c_int32), ("cache_slots", ctypes.c_int32),
                ("bytes", ctypes.c_size_t), ("min_bytes", ctypes.c_size_t),
                ("max_bytes", ctypes.c_size_t)]


class _IO(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("pos", ctypes.c_void_p), ("q_new", ctypes.c_void_p), ("k_new", ctypes.c_void_p),
                ("v_new", ctypes.c_void_p), ("pos_new", ctypes.c_void_p), ("out", ctypes.c_void_p),
                ("lse", ctypes.c_void_p), ("sel_chunk", ctypes.c_void_p),
                ("sel_group", ctypes.c_void_p), ("cache", _Cache),
                ("s_group_host", ctypes.c_void_p)]


@dataclasses.dataclass(frozen=True)
class HGAParams:
    """Method parameters (page section 3; setup table of section 6)."""
    C: int = 64
    g_s: int = 16
    F: int = 2
    L: int = 8
    K_c: int = 16
    K_g: int = 32
    rope_theta: float = 1e6
    hf_wavelength: float = 0.0   # <= 0: the chunk length C

    def c(self) -> _Params:
        return _Params(self.C, self.g_s, self.F, self.L, self.K_c, self.K_g,
                       float(self.rope_theta), float(self.hf_wavelength))


# ------------------------------------------------------------- loading --

def lib_path() -> str:
    return _LIB_PATH


def load():
    """Load libhga.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise HGAError(f"{_LIB_PATH} is missing: build it with "
                           "hierarchical_kv_routing_b200._build.build()")
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        lib.hga_build_summaries.argtypes = [P, P, P, P, P, P, P, P]
        lib.hga_route.argtypes = [P] * 10
        lib.hga_attend.argtypes = [P] * 11
        lib.hga_prefill_workspace_min.argtypes = [P, P]
        lib.hga_prefill_workspace_min.restype = ctypes.c_size_t
        lib.hga_workspace_size.argtypes = [ctypes.c_int, P, P]
        lib.hga_workspace_size.restype = ctypes.c_size_t
        lib.hga_forward.argtypes = [ctypes.c_int, P, P, P, P, ctypes.c_size_t, P]
        lib.hga_forward_prefill_noalloc.argtypes = [P, P, P, P, P, P, P, P, P]
        lib.hga_forward_prefill_noalloc.restype = ctypes.c_int
        lib.hga_status_string.argtypes = [ctypes.c_int]
        lib.hga_status_string.restype = ctypes.c_char_p
        lib.hga_last_cuda_error.restype = ctypes.c_int
        lib.hga_device_status.argtypes = [P, ctypes.c_int]
        lib.hga_device_status.restype = ctypes.c_int
        lib.hga_hostkv_link_bytes.argtypes = [P, ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_int]
        lib.hga_hostkv_link_bytes.restype = ctypes.c_int
        lib.hga_attend_backward.argtypes = [P] * 14 + [ctypes.c_size_t, P]
        lib.hga_set_test_hooks.argtypes = [ctypes.c_int, ctypes.c_ulonglong, P]
        lib.hga_set_test_hooks.restype = ctypes.c_int
        lib.hga_hostkv_plan_for.argtypes = [P, P, ctypes.c_size_t, P]
        lib.hga_hostkv_plan_for.restype = ctypes.c_int
        for f in ("hga_build_summaries", "hga_route", "hga_attend", "hga_forward",
                  "hga_attend_backward"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
        return lib


def _check(status: int, what: str):
    if status != 0:
        lib = load()
        msg = lib.hga_status_string(status).decode()
        extra = ""
        if status == 3:
            extra = f" (cuda error {lib.hga_last_cuda_error()})"
        raise HGAError(f"{what}: {msg}{extra}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None) -> ctypes.c_void_p:
    """The stream a call is enqueued on: the given one, or the current stream
    of the call's device.  A given stream must belong to that device."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise HGAError(f"stream is on {stream.device}, the call's tensors are on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on(device):
    """Make the call's device current while the library runs (the library
    launches on the current device and looks up per-device state there)."""
    return torch.cuda.device(device)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return _F32
    if t.dtype == torch.bfloat16:
        return _BF16
    raise HGAError(f"unsupported dtype {t.dtype}: float32 or bfloat16")


def _need(t: torch.Tensor, name: str, shape=None, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise HGAError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise HGAError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise HGAError(f"{name} is on {t.device}, the call's tensors are on {device}")
    if not t.is_contiguous():
        raise HGAError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise HGAError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise HGAError(f"{name} has dtype {t.dtype}, expected {dtype}")


def _dims(B, T, Hq, Hkv, D, dtype_code) -> _Dims:
    return _Dims(B, T, Hq, Hkv, D, dtype_code)


# --------------------------------------------------------------- calls --

def hga_build_summaries(k_raw: torch.Tensor, pos: torch.Tensor, params: HGAParams, *,
                        k_rot: Optional[torch.Tensor] = None, s_chunk=None, s_group=None,
                        want_k_rot: bool = True, stream=None):
    """Stage 1.  k_raw [B,T,Hkv,D] -> (k_rot [B,T,Hkv,D] or None,
    s_chunk [B,Hkv,T/C,D] f32, s_group [B,Hkv,(T/C)*(C/g_s),D] f32)."""
    lib = load()
    _need(k_raw, "k_raw")
    B, T, Hkv, D = k_raw.shape
    dev = k_raw.device
    _need(pos, "pos", (B, T), torch.int32, dev)
    NC = T // params.C
    if k_rot is None and want_k_rot:
        k_rot = torch.empty_like(k_raw)
    if s_chunk is None:
        s_chunk = torch.empty(B, Hkv, NC, D, device=dev, dtype=torch.float32)
    if s_group is None:
        s_group = torch.empty(B, Hkv, NC * (params.C // params.g_s), D, device=dev,
                              dtype=torch.float32)
    if k_rot is not None:
        _need(k_rot, "k_rot", (B, T, Hkv, D), k_raw.dtype, dev)
    _need(s_chunk, "s_chunk", (B, Hkv, NC, D), torch.float32, dev)
    _need(s_group, "s_group", (B, Hkv, NC * (params.C // params.g_s), D), torch.float32, dev)
    dims = _dims(B, T, Hkv, Hkv, D, _dtype_code(k_raw))
    pc = params.c()
    with _on(dev):
        st = lib.hga_build_summaries(ctypes.byref(dims), ctypes.byref(pc), _ptr(k_raw), _ptr(pos),
                                     _ptr(k_rot), _ptr(s_chunk), _ptr(s_group),
                                     _stream(stream, dev))
    _check(st, "hga_build_summaries")
    return k_rot, s_chunk, s_group


def hga_route(q: torch.Tensor, pos: torch.Tensor, s_chunk: torch.Tensor, s_group: torch.Tensor,
              params: HGAParams, *, sel_chunk=None, sel_group=None, q_rot=None, stream=None):
    """Stage 2.  q [B,T,Hq,D] -> sel_chunk [B,NB,Hkv,K_c], sel_group [B,NB,Hkv,K_g].
    q_rot (bf16 only): a [B,T,Hq,D] bf16 tensor that receives the rotated
    queries, for hga_attend's q_rot."""
    lib = load()
    _need(q, "q")
    B, T, Hq, D = q.shape
    dev = q.device
    Hkv = s_chunk.shape[1]
    _need(pos, "pos", (B, T), torch.int32, dev)
    _need(s_chunk, "s_chunk", (B, Hkv, T // params.C, D), torch.float32, dev)
    _need(s_group, "s_group", (B, Hkv, (T // params.C) * (params.C // params.g_s), D),
          torch.float32, dev)
    NB = (T + params.C - 1) // params.C
    if sel_chunk is None:
        sel_chunk = torch.empty(B, NB, Hkv, params.K_c, device=q.device, dtype=torch.int32)
    if sel_group is None:
        sel_group = torch.empty(B, NB, Hkv, params.K_g, device=q.device, dtype=torch.int32)
    _need(sel_chunk, "sel_chunk", (B, NB, Hkv, params.K_c), torch.int32, dev)
    _need(sel_group, "sel_group", (B, NB, Hkv, params.K_g), torch.int32, dev)
    if q_rot is not None:
        _need(q_rot, "q_rot", (B, T, Hq, D), torch.bfloat16, dev)
    dims = _dims(B, T, Hq, Hkv, D, _dtype_code(q))
    pc = params.c()
    with _on(dev):
        st = lib.hga_route(ctypes.byref(dims), ctypes.byref(pc), _ptr(q), _ptr(pos), _ptr(s_chunk),
                           _ptr(s_group), _ptr(sel_chunk), _ptr(sel_group), _ptr(q_rot),
                           _stream(stream, dev))
    _check(st, "hga_route")
    return sel_chunk, sel_group


def hga_attend(q: torch.Tensor, pos: torch.Tensor, k_rot: torch.Tensor, v: torch.Tensor,
               sel_group: torch.Tensor, params: HGAParams, *, out=None, want_lse: bool = False,
               lse=None, q_rot=None, stream=None):
    """Stage 3.  -> out [B,T,Hq,D] (and lse [B,Hq,T] f32 when asked).  q_rot:
    the rotated queries hga_route wrote (bf16), used instead of rotating q."""
    lib = load()
    _need(q, "q")
    B, T, Hq, D = q.shape
    dev = q.device
    Hkv = k_rot.shape[2]
    NB = (T + params.C - 1) // params.C
    _need(k_rot, "k_rot", (B, T, Hkv, D), q.dtype, dev)
    _need(v, "v", (B, T, Hkv, D), q.dtype, dev)
    _need(pos, "pos", (B, T), torch.int32, dev)
    _need(sel_group, "sel_group", (B, NB, Hkv, params.K_g), torch.int32, dev)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, Hq, T, device=q.device, dtype=torch.float32)
    _need(out, "out", (B, T, Hq, D), q.dtype, dev)
    if lse is not None:
        _need(lse, "lse", (B, Hq, T), torch.float32, dev)
    if q_rot is not None:
        _need(q_rot, "q_rot", (B, T, Hq, D), torch.bfloat16, dev)
    dims = _dims(B, T, Hq, Hkv, D, _dtype_code(q))
    pc = params.c()
    with _on(dev):
        st = lib.hga_attend(ctypes.byref(dims), ctypes.byref(pc), _ptr(q), _ptr(pos), _ptr(k_rot),
                            _ptr(v), _ptr(sel_group), _ptr(out), _ptr(lse), _ptr(q_rot),
                            _stream(stream, dev))
    _check(st, "hga_attend")
    return (out, lse) if want_lse or lse is not None else out


def hga_attend_backward(q: torch.Tensor, pos: torch.Tensor, k_rot: torch.Tensor, v: torch.Tensor,
                        sel_group: torch.Tensor, lse: torch.Tensor, d_out: torch.Tensor,
                        params: HGAParams, *, dq=None, dk=None, dv=None, workspace=None,
                        q_rot=None, stream=None):
    """Backward of stage 3 with the routed groups held fixed.  q, pos, k_rot,
    v, sel_group as given to hga_attend; lse as it returned it; d_out
    [B,T,Hq,D] the gradient of the loss with respect to its output.  Returns
    (dq [B,T,Hq,D], dk [B,T,Hkv,D], dv [B,T,Hkv,D]) in fp32, dq and dk with
    respect to the raw (pre-RoPE) q and k.  q_rot: the rotated queries the
    forward's hga_route wrote (bf16), which spares rotating q again."""
    lib = load()
    _need(q, "q")
    B, T, Hq, D = q.shape
    dev = q.device
    Hkv = k_rot.shape[2]
    NB = (T + params.C - 1) // params.C
    _need(pos, "pos", (B, T), torch.int32, dev)
    _need(k_rot, "k_rot", (B, T, Hkv, D), q.dtype, dev)
    _need(v, "v", (B, T, Hkv, D), q.dtype, dev)
    _need(sel_group, "sel_group", (B, NB, Hkv, params.K_g), torch.int32, dev)
    _need(lse, "lse", (B, Hq, T), torch.float32, dev)
    _need(d_out, "d_out", (B, T, Hq, D), q.dtype, dev)
    if q_rot is not None:
        _need(q_rot, "q_rot", (B, T, Hq, D), torch.bfloat16, dev)
    f32 = dict(device=dev, dtype=torch.float32)
    dq = torch.empty(B, T, Hq, D, **f32) if dq is None else dq
    dk = torch.empty(B, T, Hkv, D, **f32) if dk is None else dk
    dv = torch.empty(B, T, Hkv, D, **f32) if dv is None else dv
    _need(dq, "dq", (B, T, Hq, D), torch.float32, dev)
    _need(dk, "dk", (B, T, Hkv, D), torch.float32, dev)
    _need(dv, "dv", (B, T, Hkv, D), torch.float32, dev)
    dims = _dims(B, T, Hq, Hkv, D, _dtype_code(q))
    pc = params.c()
    nbytes = int(lib.hga_workspace_size(ATTEND_BACKWARD, ctypes.byref(dims), ctypes.byref(pc)))
    ws, base, avail = _workspace(nbytes, dev, workspace, zero=False)
    with _on(dev):
        st = lib.hga_attend_backward(ctypes.byref(dims), ctypes.byref(pc), _ptr(q), _ptr(pos),
                                     _ptr(k_rot), _ptr(v), _ptr(sel_group), _ptr(lse),
                                     _ptr(d_out), _ptr(q_rot), _ptr(dq), _ptr(dk), _ptr(dv),
                                     None if base is None else ctypes.c_void_p(base), avail,
                                     _stream(stream, dev))
    _check(st, "hga_attend_backward")
    return dq, dk, dv


def hga_device_status(clear: bool = True, stream=None) -> int:
    """The status the kernels recorded on the device since the last reset
    (0 = none; 4 = a bounded wait timed out; 5 = a bounds check refused an
    access).  Waits for the work queued on `stream`."""
    lib = load()
    return int(lib.hga_device_status(_stream(stream), 1 if clear else 0))


def hga_hostkv_link_bytes(clear: bool = True, stream=None) -> int:
    """Bytes the host tier's stage 3 has read over the host link since the
    last reset (sinks, windows and the routed groups its warm cache missed).
    Waits for the work queued on `stream`."""
    lib = load()
    v = ctypes.c_ulonglong(0)
    _check(lib.hga_hostkv_link_bytes(_stream(stream), ctypes.byref(v), 1 if clear else 0),
           "hga_hostkv_link_bytes")
    return int(v.value)


def hga_workspace_size(mode: int, B: int, T: int, Hq: int, Hkv: int, D: int, dtype,
                       params: HGAParams) -> int:
    lib = load()
    code = _F32 if dtype in (torch.float32, "f32") else _BF16
    dims = _dims(B, T, Hq, Hkv, D, code)
    pc = params.c()
    return int(lib.hga_workspace_size(mode, ctypes.byref(dims), ctypes.byref(pc)))


class KVCache:
    """Decode state for `capacity` tokens per sequence (caller-owned device
    memory, laid out as hga_kv_cache in include/hga.h)."""

    def __init__(self, B: int, capacity: int, Hkv: int, D: int, dtype, params: HGAParams,
                 device="cuda"):
        if capacity % params.C:
            raise HGAError("capacity must be a multiple of C")
        self.B, self.capacity, self.Hkv, self.D, self.dtype = B, capacity, Hkv, D, dtype
        self.params = params
        z = dict(device=device)
        self.k_rot = torch.zeros(B, capacity, Hkv, D, dtype=dtype, **z)
        self.v = torch.zeros(B, capacity, Hkv, D, dtype=dtype, **z)
        self.pos = torch.zeros(B, capacity, dtype=torch.int32, **z)
        self.k_open = torch.zeros(B, Hkv, params.C, D, dtype=dtype, **z)
        self.s_chunk = torch.zeros(B, Hkv, capacity // params.C, D, dtype=torch.float32, **z)
        self.s_group = torch.zeros(B, Hkv, capacity // params.g_s, D, dtype=torch.float32, **z)
        self.lens = torch.zeros(B, dtype=torch.int32, **z)

    def check_device(self, device):
        """Raise unless every cache buffer lies on `device`."""
        for name in ("k_rot", "v", "pos", "k_open", "s_chunk", "s_group", "lens"):
            t = getattr(self, name)
            if t.device != device:
                raise HGAError(f"cache.{name} is on {t.device}, the call's tensors are on {device}")

    def c(self) -> _Cache:
        return _Cache(self.capacity, self.k_rot.data_ptr(), self.v.data_ptr(), self.pos.data_ptr(),
                      self.k_open.data_ptr(), self.s_chunk.data_ptr(), self.s_group.data_ptr(),
                      self.lens.data_ptr())


def _workspace(nbytes: int, device, workspace: Optional[torch.Tensor], zero: bool):
    """(tensor kept alive for the call, 256-byte aligned base address, bytes
    usable from that base).  A caller's workspace must lie on the call's
    device and hold nbytes from its first 256-byte boundary on: the base is
    rounded up, so a buffer of exactly nbytes that does not start on such a
    boundary is refused rather than overrun."""
    if nbytes == 0:
        return None, None, 0
    if workspace is not None:
        if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda:
            raise HGAError("workspace must be a CUDA tensor")
        if workspace.device != device:
            raise HGAError(f"workspace is on {workspace.device}, the call's tensors are on {device}")
        if not workspace.is_contiguous():
            raise HGAError("workspace must be contiguous")
        w = workspace
    else:
        w = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        if zero:
            w.zero_()
    base, avail = _aligned_span(w.data_ptr(), w.numel() * w.element_size(), nbytes)
    return w, base, avail


def _aligned_span(start: int, size: int, nbytes: int):
    """(base, avail): the first 256-byte boundary at or after `start` and the
    bytes of [start, start + size) from there on; raises unless avail >= nbytes."""
    base = (start + 255) // 256 * 256
    avail = start + size - base
    if avail < nbytes:
        raise HGAError(f"workspace too small: need {nbytes} bytes from its first 256-byte "
                       f"boundary, have {max(avail, 0)}")
    return base, avail


def hga_forward_prefill(q, k, v, pos, params: HGAParams, *, cache: Optional[KVCache] = None,
                        out=None, want_lse=False, want_sel=False, workspace=None, stream=None):
    """Stages 1-3 in one call.  Returns dict(out, lse?, sel_chunk?, sel_group?)."""
    lib = load()
    _need(q, "q")
    B, T, Hq, D = q.shape
    dev = q.device
    Hkv = k.shape[2]
    _need(k, "k", (B, T, Hkv, D), q.dtype, dev)
    _need(v, "v", (B, T, Hkv, D), q.dtype, dev)
    _need(pos, "pos", (B, T), torch.int32, dev)
    NB = (T + params.C - 1) // params.C
    res = {"out": torch.empty_like(q) if out is None else out}
    _need(res["out"], "out", (B, T, Hq, D), q.dtype, dev)
    io = _IO()
    io.q, io.k, io.v, io.pos = q.data_ptr(), k.data_ptr(), v.data_ptr(), pos.data_ptr()
    io.out = res["out"].data_ptr()
    if want_lse:
        res["lse"] = torch.empty(B, Hq, T, device=dev, dtype=torch.float32)
        io.lse = res["lse"].data_ptr()
    if want_sel:
        res["sel_chunk"] = torch.empty(B, NB, Hkv, params.K_c, device=dev, dtype=torch.int32)
        res["sel_group"] = torch.empty(B, NB, Hkv, params.K_g, device=dev, dtype=torch.int32)
        io.sel_chunk = res["sel_chunk"].data_ptr()
        io.sel_group = res["sel_group"].data_ptr()
    if cache is not None:
        cache.check_device(dev)
        io.cache = cache.c()
    dims = _dims(B, T, Hq, Hkv, D, _dtype_code(q))
    pc = params.c()
    nbytes = int(lib.hga_workspace_size(PREFILL, ctypes.byref(dims), ctypes.byref(pc)))
    ws, base, avail = _workspace(nbytes, dev, workspace, zero=False)
    with _on(dev):
        st = lib.hga_forward(PREFILL, ctypes.byref(dims), ctypes.byref(pc), ctypes.byref(io),
                             None if base is None else ctypes.c_void_p(base), avail,
                             _stream(stream, dev))
    _check(st, "hga_forward(prefill)")
    return res


def hga_hostkv_plan(B: int, T: int, Hq: int, Hkv: int, D: int, params: HGAParams,
                    workspace_bytes: int = 0) -> dict:
    """How the host tier uses a workspace of workspace_bytes (0: report the
    bounds only): dict(wave_blocks, cache_slots, bytes, min_bytes, max_bytes);
    bytes is 0 when the workspace is below min_bytes."""
    lib = load()
    dims = _dims(B, T, Hq, Hkv, D, _BF16)
    pc = params.c()
    pl = _HostkvPlan()
    st = lib.hga_hostkv_plan_for(ctypes.byref(dims), ctypes.byref(pc), int(workspace_bytes),
                                 ctypes.byref(pl))
    if st not in (0, 6):
        _check(st, "hga_hostkv_plan_for")
    return {f: int(getattr(pl, f)) for f, _ in _HostkvPlan._fields_}


def hostkv_workspace_bytes(B, T, Hq, Hkv, D, params: HGAParams, *, cache_bytes=None,
                           vram_headroom=None, device="cuda") -> int:
    """Workspace size for the host tier.  cache_bytes: a budget in bytes
    (clamped to the tier's [min_bytes, max_bytes]).  vram_headroom: leave
    that many bytes of the device's currently free memory unused, the warm
    cache taking the rest up to max_bytes and shrinking down to min_bytes.
    Neither: the default size."""
    bounds = hga_hostkv_plan(B, T, Hq, Hkv, D, params)
    if cache_bytes is None and vram_headroom is None:
        return hga_workspace_size(PREFILL_HOSTKV, B, T, Hq, Hkv, D, torch.bfloat16, params)
    if cache_bytes is None:
        free, _ = torch.cuda.mem_get_info(torch.device(device))
        cache_bytes = free - int(vram_headroom) - 256
    return int(min(max(int(cache_bytes), bounds["min_bytes"]), bounds["max_bytes"]))


def hga_forward_prefill_hostkv(q, k_host, v_host, pos, params: HGAParams, *, out=None,
                               want_lse=False, want_sel=False, workspace=None,
                               cache_bytes=None, vram_headroom=None, s_group_host=None,
                               stream=None):
    """Prefill with the token K/V history in host RAM (the host-resident
    tier).  q [B,T,Hq,D] and pos [B,T] are CUDA tensors; k_host and v_host
    [B,T,Hkv,D] are pinned CPU tensors (raw keys, values).  Returns the same
    dict as hga_forward_prefill (the outputs equal that call's) plus "plan",
    the wave size and warm-cache slots the workspace gave (see
    hostkv_workspace_bytes for cache_bytes and vram_headroom; a caller's
    workspace is used at its own size).  s_group_host: a pinned CPU float32
    tensor [B, Hkv, (T//C)*(C//g_s), D] to hold the group summaries in the
    cold tier (written by stage 1, read by routing over the link)."""
    lib = load()
    _need(q, "q")
    B, T, Hq, D = q.shape
    dev = q.device
    Hkv = k_host.shape[2]
    for t, name in ((k_host, "k_host"), (v_host, "v_host")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned():
            raise HGAError(f"{name} must be a pinned CPU tensor")
        if not t.is_contiguous() or tuple(t.shape) != (B, T, Hkv, D) or t.dtype != q.dtype:
            raise HGAError(f"{name} must be contiguous {(B, T, Hkv, D)} {q.dtype}")
    _need(pos, "pos", (B, T), torch.int32, dev)
    NB = (T + params.C - 1) // params.C
    res = {"out": torch.empty_like(q) if out is None else out}
    _need(res["out"], "out", (B, T, Hq, D), q.dtype, dev)
    io = _IO()
    if s_group_host is not None:
        ng = (T // params.C) * (params.C // params.g_s)
        t = s_group_host
        if (not isinstance(t, torch.Tensor) or t.is_cuda or not t.is_pinned()
                or not t.is_contiguous() or t.dtype != torch.float32
                or tuple(t.shape) != (B, Hkv, ng, D)):
            raise HGAError(f"s_group_host must be a pinned contiguous float32 CPU tensor "
                           f"{(B, Hkv, ng, D)}")
        io.s_group_host = t.data_ptr()
    io.q, io.k, io.v, io.pos = q.data_ptr(), k_host.data_ptr(), v_host.data_ptr(), pos.data_ptr()
    io.out = res["out"].data_ptr()
    if want_lse:
        res["lse"] = torch.empty(B, Hq, T, device=dev, dtype=torch.float32)
        io.lse = res["lse"].data_ptr()
    if want_sel:
        res["sel_chunk"] = torch.empty(B, NB, Hkv, params.K_c, device=dev, dtype=torch.int32)
        res["sel_group"] = torch.empty(B, NB, Hkv, params.K_g, device=dev, dtype=torch.int32)
        io.sel_chunk = res["sel_chunk"].data_ptr()
        io.sel_group = res["sel_group"].data_ptr()
    dims = _dims(B, T, Hq, Hkv, D, _dtype_code(q))
    pc = params.c()
    if workspace is not None:
        nbytes = hga_hostkv_plan(B, T, Hq, Hkv, D, params)["min_bytes"]
    else:
        nbytes = hostkv_workspace_bytes(B, T, Hq, Hkv, D, params, cache_bytes=cache_bytes,
                                        vram_headroom=vram_headroom, device=dev)
    ws, base, avail = _workspace(nbytes, dev, workspace, zero=False)
    res["plan"] = hga_hostkv_plan(B, T, Hq, Hkv, D, params, avail)
    with _on(dev):
        st = lib.hga_forward(PREFILL_HOSTKV, ctypes.byref(dims), ctypes.byref(pc),
                             ctypes.byref(io), None if base is None else ctypes.c_void_p(base),
                             avail, _stream(stream, dev))
    _check(st, "hga_forward(prefill, host K/V)")
    return res


def hga_fill_cache(k, v, pos, cache: "KVCache", params: HGAParams, *, stream=None):
    """Fill a decode cache from a prompt's raw keys, values and positions
    (stage 1 only: rotated keys, values, positions, summaries, lens = T)."""
    lib = load()
    _need(k, "k")
    B, T, Hkv, D = k.shape
    dev = k.device
    _need(v, "v", (B, T, Hkv, D), k.dtype, dev)
    _need(pos, "pos", (B, T), torch.int32, dev)
    cache.check_device(dev)
    io = _IO()
    io.k, io.v, io.pos = k.data_ptr(), v.data_ptr(), pos.data_ptr()
    io.cache = cache.c()
    dims = _dims(B, T, Hkv, Hkv, D, _dtype_code(k))
    pc = params.c()
    with _on(dev):
        st = lib.hga_forward(PREFILL, ctypes.byref(dims), ctypes.byref(pc), ctypes.byref(io),
                             None, 0, _stream(stream, dev))
    _check(st, "hga_forward(prefill, cache fill)")
    return cache


def hga_forward_prefill_noalloc(q, k, v, pos, params: HGAParams, out: torch.Tensor, *,
                                lse: Optional[torch.Tensor] = None, stream=None):
    """The prefill path on the library's fixed 16 MiB device scratch, for
    callers that cannot allocate at call time (their device memory belongs to
    another allocator or a fixed arena).  The caller passes every buffer,
    including `out` ([B,T,Hq,D]) and optionally `lse` ([B,Hq,T] f32); this
    wrapper allocates nothing.  Shapes needing more scratch are rejected."""
    lib = load()
    _need(q, "q")
    B, T, Hq, D = q.shape
    dev = q.device
    Hkv = k.shape[2]
    _need(k, "k", (B, T, Hkv, D), q.dtype, dev)
    _need(v, "v", (B, T, Hkv, D), q.dtype, dev)
    _need(pos, "pos", (B, T), torch.int32, dev)
    _need(out, "out", (B, T, Hq, D), q.dtype, dev)
    if lse is not None:
        _need(lse, "lse", (B, Hq, T), torch.float32, dev)
    dims = _dims(B, T, Hq, Hkv, D, _dtype_code(q))
    pc = params.c()
    with _on(dev):
        st = lib.hga_forward_prefill_noalloc(ctypes.byref(dims), ctypes.byref(pc), _ptr(q),
                                             _ptr(k), _ptr(v), _ptr(pos), _ptr(out), _ptr(lse),
                                             _stream(stream, dev))
    _check(st, "hga_forward_prefill_noalloc")
    return out


def hga_forward_decode(q_new, k_new, v_new, pos_new, cache: KVCache, params: HGAParams, *,
                       out=None, want_lse=False, want_sel=False, workspace=None, stream=None):
    """One decode step per sequence.  q_new [B,Hq,D], k_new/v_new [B,Hkv,D],
    pos_new [B] int32.  `workspace` must come from decode_workspace() (zeroed
    once) when given.  Returns dict(out, lse?, sel_chunk?, sel_group?)."""
    lib = load()
    _need(q_new, "q_new")
    B, Hq, D = q_new.shape
    dev = q_new.device
    Hkv = k_new.shape[1]
    _need(k_new, "k_new", (B, Hkv, D), q_new.dtype, dev)
    _need(v_new, "v_new", (B, Hkv, D), q_new.dtype, dev)
    _need(pos_new, "pos_new", (B,), torch.int32, dev)
    cache.check_device(dev)
    res = {"out": torch.empty_like(q_new) if out is None else out}
    _need(res["out"], "out", (B, Hq, D), q_new.dtype, dev)
    io = _IO()
    io.q_new, io.k_new, io.v_new = q_new.data_ptr(), k_new.data_ptr(), v_new.data_ptr()
    io.pos_new = pos_new.data_ptr()
    io.out = res["out"].data_ptr()
    if want_lse:
        res["lse"] = torch.empty(B, Hq, device=dev, dtype=torch.float32)
        io.lse = res["lse"].data_ptr()
    if want_sel:
        res["sel_chunk"] = torch.empty(B, Hkv, params.K_c, device=dev, dtype=torch.int32)
        res["sel_group"] = torch.empty(B, Hkv, params.K_g, device=dev, dtype=torch.int32)
        io.sel_chunk = res["sel_chunk"].data_ptr()
        io.sel_group = res["sel_group"].data_ptr()
    io.cache = cache.c()
    dims = _dims(B, cache.capacity, Hq, Hkv, D, _dtype_code(q_new))
    pc = params.c()
    nbytes = int(lib.hga_workspace_size(DECODE, ctypes.byref(dims), ctypes.byref(pc)))
    ws, base, avail = _workspace(nbytes, dev, workspace, zero=True)
    with _on(dev):
        st = lib.hga_forward(DECODE, ctypes.byref(dims), ctypes.byref(pc), ctypes.byref(io),
                             None if base is None else ctypes.c_void_p(base), avail,
                             _stream(stream, dev))
    _check(st, "hga_forward(decode)")
    return res


def decode_workspace(B, capacity, Hq, Hkv, D, dtype, params: HGAParams, device="cuda"):
    """A zero-filled decode workspace (reusable across steps)."""
    n = hga_workspace_size(DECODE, B, capacity, Hq, Hkv, D, dtype, params)
    return torch.zeros(max(n, 1) + 256, dtype=torch.uint8, device=device)


def hga_forward(mode: int, *args, **kw):
    """hga_forward(PREFILL, q, k, v, pos, params, ...),
    hga_forward(DECODE, q_new, k_new, v_new, pos_new, cache, params, ...) or
    hga_forward(PREFILL_HOSTKV, q, k_host, v_host, pos, params, ...)."""
    if mode == PREFILL:
        return hga_forward_prefill(*args, **kw)
    if mode == DECODE:
        return hga_forward_decode(*args, **kw)
    if mode == PREFILL_HOSTKV:
        return hga_forward_prefill_hostkv(*args, **kw)
    raise HGAError(f"unknown mode {mode}")
