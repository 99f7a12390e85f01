"""The C-ABI library loads and exports every entry point that include/*.h
declares; the binding fails loudly without it; the product path never uses
the oracle.  No GPU needed (nothing here launches a kernel)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"^\s*(?:[A-Za-z_][\w\s\*]*?)\b(moe_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ["moe_pack_weights", "moe_unpack_weights", "moe_route", "moe_sort", "moe_forward"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    import fp4_routed_mixture_b200 as m
    lib = ctypes.CDLL(m.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert sorted(m.SYMBOLS) == declared_functions()


def test_size_queries_without_gpu():
    import fp4_routed_mixture_b200 as m
    assert m.moe_packed_bytes(4096, 2048, 256) == 256 + 256 * (2 * 2048 * 4096 + 4096 * 2048) * 17 // 32
    assert m.moe_workspace_bytes(8, 4096, 2048, 256, 6) > 0
    with pytest.raises(m.MoeError):
        m.moe_packed_bytes(4096, 2000, 256)


def test_binding_fails_loudly_without_library(monkeypatch):
    import fp4_routed_mixture_b200.binding as b
    monkeypatch.setattr(b, "LIB_PATH", os.path.join(ROOT, "does", "not", "exist.so"))
    with pytest.raises(ImportError):
        b._load()


def test_product_path_does_not_use_the_oracle():
    pkg = os.path.join(ROOT, "fp4_routed_mixture_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.*"), recursive=True):
        if path.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
            src = open(path).read()
            assert not re.search(r"(import\s+oracle|from\s+oracle|liboracle|oracle/)", src), path
