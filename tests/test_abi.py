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


def test_layer_tables_point_into_the_layer_workspace():
    # pure pointer arithmetic: a fake workspace address is never dereferenced
    import fp4_routed_mixture_b200 as m
    lib = m.lib
    for (T, H, I, E, k) in [(8, 4096, 2048, 256, 6), (1, 128, 128, 1, 1), (31, 128, 128, 1024, 16)]:
        d = m.binding.moe_dims(T, H, I, E, k)
        base = 1 << 32
        ptrs = [ctypes.c_void_p() for _ in range(5)]
        assert lib.moe_layer_tables(ctypes.byref(d), ctypes.c_void_p(base), *[ctypes.byref(p) for p in ptrs]) == 0
        off = [p.value - base for p in ptrs]
        P = T * k
        sizes = [4 * P, 4 * P, 4 * P, 4 * P, 4 * (E + 1)]   # idx, gates, perm, pos, offsets
        fwd = m.moe_workspace_bytes(T, H, I, E, k)
        total = m.moe_layer_workspace_bytes(T, H, I, E, k)
        assert off[0] >= 256                                 # after the layer's error word
        assert total >= off[4] + sizes[4] + fwd              # the forward workspace follows the tables
        for o, sz, nxt in zip(off, sizes, off[1:] + [total]):
            assert o % 256 == 0 and o + sz <= nxt
        # the tables' offsets do not depend on the tensor-core threshold
        old = m.moe_get_option(m.MOE_OPT_TC_MIN_ROWS)
        m.moe_set_option(m.MOE_OPT_TC_MIN_ROWS, 1)
        try:
            ptrs2 = [ctypes.c_void_p() for _ in range(5)]
            lib.moe_layer_tables(ctypes.byref(d), ctypes.c_void_p(base), *[ctypes.byref(p) for p in ptrs2])
            assert [p.value for p in ptrs2] == [p.value for p in ptrs]
        finally:
            m.moe_set_option(m.MOE_OPT_TC_MIN_ROWS, old)
    null = ctypes.c_void_p()
    assert m.binding.STATUS[lib.moe_layer_tables(ctypes.byref(d), None, *[ctypes.byref(null)] * 5)] == "MOE_ERR_INVALID_ARG"


def test_workspace_sized_for_the_rows_each_gemm_owns():
    # the fp64 accumulators and h codes of the streaming GEMM are sized for at
    # most E * (threshold - 1) rows once T reaches the threshold, so the
    # skewed prefill's workspace stays far below one sized for every pair
    import fp4_routed_mixture_b200 as m
    T, H, I, E, k = 16384, 4096, 2048, 256, 6
    P = T * k
    every_pair = 8 * P * (2 * I + H)                    # fp64 sums of every pair
    ws = m.moe_workspace_bytes(T, H, I, E, k)
    assert ws < 6e9 and ws + every_pair * 0.8 > every_pair
    old = m.moe_get_option(m.MOE_OPT_TC_MIN_ROWS)
    try:
        m.moe_set_option(m.MOE_OPT_TC_MIN_ROWS, 1)      # every expert on tensor cores
        ws1 = m.moe_workspace_bytes(T, H, I, E, k)
        m.moe_set_option(m.MOE_OPT_TC_MIN_ROWS, 64)
        ws64 = m.moe_workspace_bytes(T, H, I, E, k)
    finally:
        m.moe_set_option(m.MOE_OPT_TC_MIN_ROWS, old)
    per_stream_row = 8 * (2 * I + H) + I + 4 * (I // 32)
    assert ws1 < ws < ws64
    assert abs((ws64 - ws1) - E * 63 * per_stream_row) <= 8 * 256
    # below the threshold every row may be a streaming row
    assert m.moe_workspace_bytes(8, H, I, E, k) >= 8 * k * per_stream_row
