"""The oracle and the CUDA library share no code: the oracle's C file
includes only the C standard library and POSIX threads, its Python wrapper
imports neither the library nor the input generators' consumers, the
library's sources never include or import the oracle, and the seeded input
module imports neither.  The product path fails loudly without its built
library (no fallback)."""
import os
import re

import pytest

import hierarchical_kv_routing_b200 as hga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "hierarchical_kv_routing_b200")


def _read(*parts):
    return open(os.path.join(ROOT, *parts)).read()


def _files(top, exts):
    for d, _, fs in os.walk(top):
        for f in fs:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_oracle_includes_only_standard_headers():
    inc = re.findall(r'#include\s*[<"]([^>"]+)[>"]', _read("oracle", "hga_oracle.c"))
    assert set(inc) <= {"math.h", "pthread.h", "stdint.h", "stdlib.h", "string.h"}


def test_oracle_wrapper_imports_no_library_code():
    src = _read("oracle", "__init__.py")
    assert "hierarchical_kv_routing_b200" not in src and "workloads" not in src
    assert "libhga" not in src


def test_library_never_reaches_the_oracle():
    for path in _files(PKG, (".cu", ".cuh", ".h", ".py")):
        if os.sep + "_build" + os.sep in path:
            continue
        src = open(path).read()
        assert not re.search(r'#include\s*[<"][^>"]*oracle', src), path
        assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), path
        assert "liboracle" not in src and "hga_oracle" not in src, path
    assert "oracle" not in _read("include", "hga.h")


def test_input_generators_hold_no_library_or_oracle_code():
    src = _read("workloads", "__init__.py")
    assert not re.search(r"^\s*(import|from)\s+(oracle|hierarchical_kv_routing_b200)", src, re.M)


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(hga, "_lib", None)
    monkeypatch.setattr(hga, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "libhga.so"))
    with pytest.raises(hga.HGAError, match="missing"):
        hga.load()
