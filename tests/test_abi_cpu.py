"""CPU-only checks of the boundary: the library loads and exports every symbol
include/idx.h declares; the product path never touches the oracle; a missing
library is an error, not a fallback."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "idx.h")
PKG = os.path.join(ROOT, "page_scoring_top_b200")


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"^IDX_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, re.M)


@pytest.fixture(scope="module")
def libidx():
    from page_scoring_top_b200 import build
    build.build()
    return ctypes.CDLL(build.LIB)


def test_header_declares_the_abi():
    syms = set(declared_symbols())
    assert {"idx_init", "idx_destroy", "centroid_score", "topk_select", "score_topk_fused",
            "idx_get_status", "idx_strerror"} <= syms


def test_library_exports_every_declared_symbol(libidx):
    for name in declared_symbols():
        assert hasattr(libidx, name), name


def test_binding_covers_every_declared_symbol():
    from page_scoring_top_b200 import binding
    assert set(declared_symbols()) == set(binding.SIGNATURES)


def test_strerror_needs_no_gpu(libidx):
    libidx.idx_strerror.restype = ctypes.c_char_p
    assert libidx.idx_strerror(0) == b"ok"
    assert b"limits" in libidx.idx_strerror(-3)


def test_init_rejects_bad_limits_without_touching_a_gpu(libidx):
    h = ctypes.c_void_p()
    assert libidx.idx_init(ctypes.byref(h), 0, 0, 10, 10) == -1
    assert libidx.idx_init(ctypes.byref(h), 0, 10, 10, 4096) == -2
    assert libidx.idx_init(None, 0, 10, 10, 10) == -1


def test_product_never_imports_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text, f


def test_missing_library_fails_loudly(monkeypatch):
    from page_scoring_top_b200 import binding
    monkeypatch.setattr(binding, "LIB_PATH", "/nonexistent/libidx.so")
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError):
        binding.lib()
