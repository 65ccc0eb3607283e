"""The C-ABI library loads and exports every symbol include/hga.h declares,
and its host-side argument checks answer without touching a GPU."""
import ctypes
import os
import re

import pytest

import hierarchical_kv_routing_b200 as hga
from hierarchical_kv_routing_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return hga.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hga.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hga_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert {"hga_build_summaries", "hga_route", "hga_attend", "hga_forward",
            "hga_workspace_size", "hga_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def _dims(**kw):
    d = dict(B=1, T=1024, Hq=2, Hkv=1, D=64, dtype=0)
    d.update(kw)
    return hga._Dims(**d)


def test_status_strings(lib):
    for code in range(7):
        assert lib.hga_status_string(code)


def test_workspace_size_host_only(lib):
    p = hga.HGAParams(F=2, L=2, K_c=4, K_g=8, rope_theta=1e4).c()
    d = _dims()
    n = lib.hga_workspace_size(0, ctypes.byref(d), ctypes.byref(p))
    # K_rot + chunk + group summaries + selections, each 256-byte padded
    assert n >= 1024 * 64 * 4 + 16 * 64 * 4 + 64 * 64 * 4 + 16 * (4 + 8) * 4


@pytest.mark.parametrize("bad,code", [
    (dict(D=96), 2), (dict(Hq=3, Hkv=2), 1), (dict(dtype=7), 1), (dict(B=0), 1),
    (dict(B=65536, T=64), 2), (dict(Hq=65536, Hkv=65536), 2), (dict(B=2, T=1 << 30), 2)])
def test_bad_dims_rejected_before_launch(lib, bad, code):
    p = hga.HGAParams(rope_theta=1e4).c()
    d = _dims(**bad)
    io = hga._IO()
    st = lib.hga_forward(0, ctypes.byref(d), ctypes.byref(p), ctypes.byref(io), None, 0, None)
    assert st == code


@pytest.mark.parametrize("bad,code", [
    (dict(C=32), 2), (dict(g_s=5), 1), (dict(K_c=-1), 1), (dict(rope_theta=0.5), 1),
    (dict(K_g=5000), 2)])
def test_bad_params_rejected_before_launch(lib, bad, code):
    kw = dict(rope_theta=1e4)
    kw.update(bad)
    p = hga.HGAParams(**kw).c()
    d = _dims()
    io = hga._IO()
    st = lib.hga_build_summaries(ctypes.byref(d), ctypes.byref(p), None, None, None, None, None,
                                 None)
    assert st == code


def test_null_buffers_rejected(lib):
    p = hga.HGAParams(rope_theta=1e4).c()
    d = _dims()
    st = lib.hga_route(ctypes.byref(d), ctypes.byref(p), None, None, None, None, None, None, None,
                       None)
    assert st == 1
    io = hga._IO()
    st = lib.hga_forward(0, ctypes.byref(d), ctypes.byref(p), ctypes.byref(io), None, 0, None)
    assert st == 1  # null inputs are rejected before the workspace is looked at


def test_binding_fails_loudly_without_cuda():
    import torch
    if torch.cuda.is_available():
        pytest.skip("CUDA present")
    with pytest.raises(hga.HGAError):
        hga.hga_build_summaries(torch.zeros(1, 64, 1, 64), torch.zeros(1, 64, dtype=torch.int32),
                                hga.HGAParams())


def test_hostkv_mode_host_checks(lib):
    """HGA_PREFILL_HOSTKV: workspace sized on the host; fp32 and missing
    buffers rejected before anything is launched (the workspace pointer
    below is never dereferenced)."""
    p = hga.HGAParams(F=2, L=8, K_c=16, K_g=32, rope_theta=1e6).c()
    d = _dims(T=4096, Hq=32, Hkv=4, D=128, dtype=1)
    n = lib.hga_workspace_size(2, ctypes.byref(d), ctypes.byref(p))
    # the K and V row spaces dominate: two staging buffers (sinks and the
    # window of a 32-block wave) and the group cache (every group of the
    # 64 chunks here, fewer than two waves' worth of routed groups)
    groups = min(64 * (64 // 16), 2 * 32 * 32)
    rows = 2 * (2 * 64 + (32 + 8) * 64) + groups * 16
    assert n >= 2 * rows * 4 * 128 * 2
    io = hga._IO()
    fake = ctypes.c_void_p(1 << 20)
    st = lib.hga_forward(2, ctypes.byref(d), ctypes.byref(p), ctypes.byref(io), fake, n, None)
    assert st == 1
    st = lib.hga_forward(2, ctypes.byref(d), ctypes.byref(p), ctypes.byref(io), None, 0, None)
    assert st == 6
    d32 = _dims(T=4096, Hq=32, Hkv=4, D=128, dtype=0)
    n32 = lib.hga_workspace_size(2, ctypes.byref(d32), ctypes.byref(p))
    st = lib.hga_forward(2, ctypes.byref(d32), ctypes.byref(p), ctypes.byref(io), fake, n32, None)
    assert st == 2


def test_hostkv_link_bytes_checks_its_pointer(lib):
    """hga_hostkv_link_bytes refuses a null result pointer before any CUDA call."""
    lib.hga_hostkv_link_bytes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    lib.hga_hostkv_link_bytes.restype = ctypes.c_int
    assert lib.hga_hostkv_link_bytes(None, None, 0) == 1     # HGA_ERR_INVALID_ARG


def test_decode_mode_host_checks(lib):
    """HGA_DECODE: the workspace, the step's inputs and every cache buffer are
    checked on the host; a cache whose capacity is not dims.T and a
    misaligned row are refused before anything is launched (the fake pointers
    below are never dereferenced, and no call here is valid enough to launch)."""
    by = ctypes.byref
    p = hga.HGAParams(F=2, L=8, K_c=16, K_g=32, rope_theta=1e6).c()
    d = _dims(B=2, T=4096, Hq=32, Hkv=4, D=128, dtype=1)
    n = lib.hga_workspace_size(1, by(d), by(p))
    assert n > 0
    ws = ctypes.c_void_p(1 << 20)
    io = hga._IO()
    assert lib.hga_forward(1, by(d), by(p), by(io), None, 0, None) == 6       # no workspace
    assert lib.hga_forward(1, by(d), by(p), by(io), ws, n - 1, None) == 6     # too small
    assert lib.hga_forward(1, by(d), by(p), by(io), ws, n, None) == 1         # no inputs
    A = 1 << 24
    for f in ("q_new", "k_new", "v_new", "pos_new", "out"):
        setattr(io, f, A)
    assert lib.hga_forward(1, by(d), by(p), by(io), ws, n, None) == 1         # no cache
    io.cache.capacity = 4096 - 64
    for f in ("k_rot", "v", "pos", "k_open", "s_chunk", "s_group", "lens"):
        setattr(io.cache, f, A)
    assert lib.hga_forward(1, by(d), by(p), by(io), ws, n, None) == 1         # capacity != T
    io.cache.capacity = 4096
    io.out = A + 8
    assert lib.hga_forward(1, by(d), by(p), by(io), ws, n, None) == 1         # misaligned out


def test_prefill_cache_fill_host_checks(lib):
    """HGA_PREFILL filling a decode cache: a capacity below T or not a whole
    number of chunks, and a cache beyond the 32-bit row limit, are refused
    before any launch (fake pointers, never dereferenced)."""
    by = ctypes.byref
    p = hga.HGAParams(F=2, L=8, K_c=16, K_g=32, rope_theta=1e6).c()
    d = _dims(B=2, T=4096, Hq=32, Hkv=4, D=128, dtype=1)
    A = 1 << 24
    io = hga._IO()
    for f in ("k", "v", "pos"):                 # cache fill only: no q, no out
        setattr(io, f, A)
    for f in ("k_rot", "v", "pos", "k_open", "s_chunk", "s_group", "lens"):
        setattr(io.cache, f, A)
    io.cache.capacity = 4096 - 64
    assert lib.hga_forward(0, by(d), by(p), by(io), None, 0, None) == 1       # below T
    io.cache.capacity = 4096 + 32
    assert lib.hga_forward(0, by(d), by(p), by(io), None, 0, None) == 1       # not whole chunks
    io.cache.capacity = 1 << 30
    assert lib.hga_forward(0, by(d), by(p), by(io), None, 0, None) == 2       # B*capacity >= 2^31


def test_noalloc_rejects_oversized_shapes_on_the_host(lib):
    """The no-allocation prefill refuses a shape whose scratch exceeds its
    fixed 16 MiB before any CUDA call (fake pointers, never dereferenced)."""
    by = ctypes.byref
    p = hga.HGAParams(F=2, L=8, K_c=16, K_g=32, rope_theta=1e6).c()
    big = _dims(B=1, T=32768, Hq=32, Hkv=4, D=128, dtype=1)
    assert lib.hga_workspace_size(0, by(big), by(p)) > 16 << 20
    A = ctypes.c_void_p(1 << 24)
    st = lib.hga_forward_prefill_noalloc(by(big), by(p), A, A, A, A, A, None, None)
    assert st == 6


@pytest.mark.parametrize("start,size,need,ok", [
    (0x7f0000000000, 4096, 4096, True),          # aligned, exact size
    (0x7f0000000010, 4096, 4096, False),         # unaligned slice of exactly nbytes
    (0x7f0000000010, 4096 + 240, 4096, True),    # unaligned, enough after the boundary
    (0x7f00000000f0, 4096 + 15, 4096, False),    # one byte short after rounding up
])
def test_workspace_span_accounts_for_alignment(start, size, need, ok):
    """A caller's workspace is used from its first 256-byte boundary, and the
    bytes passed to the library are those left from there, so a buffer that
    starts off a boundary is refused unless the rest still holds nbytes."""
    if ok:
        base, avail = hga._aligned_span(start, size, need)
        assert base % 256 == 0 and base >= start and avail >= need
        assert base + avail == start + size
    else:
        with pytest.raises(hga.HGAError, match="workspace too small"):
            hga._aligned_span(start, size, need)


def test_hostkv_plan_bounds_and_monotone_growth(lib):
    """The host tier's plan for a workspace size (host-only): the smallest
    plan is one block per wave with a two-wave cache, the default is 32-block
    waves with two waves' worth of slots, a larger workspace only adds slots
    (up to every group), a smaller one shrinks the wave; below the minimum
    the call reports HGA_ERR_WORKSPACE."""
    hp = hga.HGAParams(C=64, g_s=16, F=2, L=8, K_c=16, K_g=32, rope_theta=1e6)
    b = hga.hga_hostkv_plan(1, 65536, 32, 4, 128, hp)
    assert b["bytes"] == 0 and b["min_bytes"] < b["max_bytes"]
    lo = hga.hga_hostkv_plan(1, 65536, 32, 4, 128, hp, b["min_bytes"])
    assert (lo["wave_blocks"], lo["cache_slots"], lo["bytes"]) == (1, 64, b["min_bytes"])
    assert hga.hga_hostkv_plan(1, 65536, 32, 4, 128, hp, b["min_bytes"] - 1)["bytes"] == 0
    d = hga.hga_workspace_size(hga.PREFILL_HOSTKV, 1, 65536, 32, 4, 128, "bf16", hp)
    mid = hga.hga_hostkv_plan(1, 65536, 32, 4, 128, hp, d)
    assert (mid["wave_blocks"], mid["cache_slots"], mid["bytes"]) == (32, 2 * 32 * 32, d)
    top = hga.hga_hostkv_plan(1, 65536, 32, 4, 128, hp, b["max_bytes"])
    assert (top["wave_blocks"], top["cache_slots"]) == (32, 65536 // 16)
    prev = None
    for nb in range(b["min_bytes"], b["max_bytes"] + 1, (b["max_bytes"] - b["min_bytes"]) // 37):
        pl = hga.hga_hostkv_plan(1, 65536, 32, 4, 128, hp, nb)
        assert 0 < pl["bytes"] <= nb
        assert pl["cache_slots"] >= 2 * pl["wave_blocks"] * 32
        if prev is not None:
            assert (pl["wave_blocks"], pl["cache_slots"]) >= (prev["wave_blocks"], prev["cache_slots"])
        prev = pl
