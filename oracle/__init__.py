"""ctypes wrapper of the CPU oracle (``moe_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
CPU-baseline leg of the benchmark, never by the product path.  It shares no
code with the CUDA library.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_SRCS = [_SRC, os.path.join(_HERE, "fp8_oracle.cpp")]
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, IEEE arithmetic, no contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or any(os.path.getmtime(_LIB) < os.path.getmtime(f) for f in _SRCS):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp] + _SRCS + ["-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i32, i64, vp, d, f = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_double, ctypes.c_float
        _lib.orc_e2m1.argtypes, _lib.orc_e2m1.restype = [i32], d
        _lib.orc_e8m0.argtypes, _lib.orc_e8m0.restype = [i32], d
        _lib.orc_exp.argtypes, _lib.orc_exp.restype = [f], f
        _lib.orc_swiglu.argtypes, _lib.orc_swiglu.restype = [f, f], f
        _lib.orc_bf16_from_double.argtypes, _lib.orc_bf16_from_double.restype = [d], ctypes.c_uint16
        _lib.orc_exp_array.argtypes = [vp, vp, i64]
        _lib.orc_quant_rows.argtypes = [vp, i64, i32, vp, vp]
        _lib.orc_quant_x.argtypes = [vp, i32, i32, vp, vp, i32]
        _lib.orc_route.argtypes = [vp, i32, i32, i32, vp, vp]
        _lib.orc_router_logits.argtypes = [vp, vp, vp, i32, i32, i32, vp, i32]
        _lib.orc_sort.argtypes = [vp, i32, i32, i32, vp, vp, vp, vp]
        _lib.orc_sort.restype = i32
        _lib.orc_row_dot.argtypes, _lib.orc_row_dot.restype = [vp, vp, vp, i32], d
        _lib.orc_row_dot_fixed.argtypes, _lib.orc_row_dot_fixed.restype = [vp, vp, vp, i32, vp], i32
        _lib.orc_rows_dot.argtypes = [vp, i32, vp, vp, vp, vp, i64, vp, vp, vp, i32]
        _lib.orc_forward.argtypes = [i32] * 5 + [vp] * 6 + [vp] * 12 + [i32]
        _lib.orc_forward.restype = i32
        _lib.orc_forward_tokens.argtypes = [i32] * 5 + [vp] * 6 + [vp, i32] + [vp] * 7 + [i32]
        _lib.orc_forward_tokens.restype = i32
        _lib.orc_forward_dense.argtypes = [i32] * 5 + [vp] * 6 + [vp, vp, i32]
        _lib.orc_forward_dense.restype = i32
        _lib.orc_e4m3.argtypes, _lib.orc_e4m3.restype = [i32], d
        _lib.orc_e4m3_code.argtypes, _lib.orc_e4m3_code.restype = [d], i32
        _lib.orc_fp8_quant_act.argtypes = [vp, i32, i32, vp, vp, i32]
        _lib.orc_fp8_linear.argtypes = [vp, vp, vp, vp, i32, i32, i32, vp, vp, vp, i32]
    return _lib


def nthreads() -> int:
    return max(1, os.cpu_count() or 1)


def _p(a):
    if a is None:
        return None
    assert isinstance(a, np.ndarray) and a.flags["C_CONTIGUOUS"], "need a C-contiguous array"
    return a.ctypes.data


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ---- elementwise definitions -------------------------------------------------

def e2m1(code: int) -> float:
    return _L().orc_e2m1(code)


def e8m0(s: int) -> float:
    return _L().orc_e8m0(s)


def exp_f32(x) -> np.ndarray:
    x = _c(x, np.float32).ravel()
    y = np.empty_like(x)
    _L().orc_exp_array(_p(x), _p(y), x.size)
    return y


def swiglu(g: float, u: float) -> float:
    return _L().orc_swiglu(g, u)


def bf16_from_double(v: float) -> int:
    return int(_L().orc_bf16_from_double(v))


def quant_rows(v: np.ndarray):
    v = _c(v, np.float32)
    rows, cols = v.shape
    q = np.empty((rows, cols), np.int8)
    s = np.empty(rows, np.float32)
    _L().orc_quant_rows(_p(v), rows, cols, _p(q), _p(s))
    return q, s


def quant_x(x_bf16: np.ndarray):
    x = _c(x_bf16, np.uint16)
    T, H = x.shape
    q = np.empty((T, H), np.int8)
    s = np.empty(T, np.float32)
    _L().orc_quant_x(_p(x), T, H, _p(q), _p(s), nthreads())
    return q, s


def router_logits(x_bits: np.ndarray, wr: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """S[t,e] = sum_h x[t,h] * wr[e,h] (+ bias[e]) in fp64; x as raw bf16 bits."""
    x = _c(x_bits, np.uint16)
    w = _c(wr, np.float32)
    T, H = x.shape
    E = w.shape[0]
    assert w.shape[1] == H
    b = None if bias is None else _c(bias, np.float32)
    out = np.empty((T, E), np.float64)
    _L().orc_router_logits(_p(x), _p(w), None if b is None else _p(b), T, H, E, _p(out), nthreads())
    return out


def route(logits: np.ndarray, k: int):
    l = _c(logits, np.float32)
    T, E = l.shape
    idx = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float64)
    _L().orc_route(_p(l), T, E, k, _p(idx), _p(gates))
    return idx, gates


def sort(idx: np.ndarray, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    P = T * k
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(P, np.int32)
    pos = np.empty(P, np.int32)
    rc = _L().orc_sort(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(pos))
    if rc != 0:
        raise ValueError("expert id outside [0, E)")
    return counts, offsets, perm, pos


def row_dot(q, codes, scales) -> float:
    q, codes, scales = _c(q, np.int8), _c(codes, np.uint8), _c(scales, np.uint8)
    K = q.size
    assert codes.size == K // 2 and scales.size == K // 32
    return _L().orc_row_dot(_p(q), _p(codes), _p(scales), K)


def row_dot_fixed(q, codes, scales):
    """int64 fixed-point variant; returns None outside its exact range."""
    q, codes, scales = _c(q, np.int8), _c(codes, np.uint8), _c(scales, np.uint8)
    out = ctypes.c_double()
    rc = _L().orc_row_dot_fixed(_p(q), _p(codes), _p(scales), q.size, ctypes.byref(out))
    return None if rc else out.value


def rows_dot(q2d, qrow, codes2d, scales2d, wrow, fixed: bool = True):
    """out[r] = dot(q2d[qrow[r]], weight row wrow[r]); both references."""
    q2d, codes2d, scales2d = _c(q2d, np.int8), _c(codes2d, np.uint8), _c(scales2d, np.uint8)
    qrow, wrow = _c(qrow, np.int32), _c(wrow, np.int64)
    K = q2d.shape[1]
    n = qrow.size
    out = np.empty(n, np.float64)
    outf = np.empty(n, np.float64) if fixed else None
    ok = np.empty(n, np.int32) if fixed else None
    _L().orc_rows_dot(_p(q2d), K, _p(qrow), _p(codes2d), _p(scales2d), _p(wrow), n, _p(out),
                      _p(outf), _p(ok), nthreads())
    return (out, outf, ok) if fixed else out


# ---- the layer ------------------------------------------------------------------

def forward(x, logits, w1_codes, w1_scales, w2_codes, w2_scales, k: int, want_Y: bool = False):
    """All outputs of the layer; per-pair values indexed by pair id t*k+j."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    w1c, w1s, w2c, w2s = (_c(a, np.uint8) for a in (w1_codes, w1_scales, w2_codes, w2_scales))
    T, H = x.shape
    E = logits.shape[1]
    I = w2c.shape[2] * 2
    P = T * k
    o = dict(idx=np.empty((T, k), np.int32), gates=np.empty((T, k), np.float64),
             counts=np.empty(E, np.int32), offsets=np.empty(E + 1, np.int32),
             perm=np.empty(P, np.int32), pos=np.empty(P, np.int32),
             xq=np.empty((T, H), np.int8), sx=np.empty(T, np.float32),
             hq=np.empty((P, I), np.int8), sh=np.empty(P, np.float32),
             Y=np.empty((P, H), np.float32) if want_Y else None,
             y=np.empty((T, H), np.uint16))
    rc = _L().orc_forward(T, H, I, E, k, _p(x), _p(logits), _p(w1c), _p(w1s), _p(w2c), _p(w2s),
                          _p(o["idx"]), _p(o["gates"]), _p(o["counts"]), _p(o["offsets"]),
                          _p(o["perm"]), _p(o["pos"]), _p(o["xq"]), _p(o["sx"]), _p(o["hq"]),
                          _p(o["sh"]), _p(o["Y"]), _p(o["y"]), nthreads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    if not want_Y:
        del o["Y"]
    return o


def forward_tokens(x, logits, w1_codes, w1_scales, w2_codes, w2_scales, k: int, tokens):
    """The layer's values for the listed tokens only (sampled full-size checks)."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    w1c, w1s, w2c, w2s = (_c(a, np.uint8) for a in (w1_codes, w1_scales, w2_codes, w2_scales))
    tok = _c(tokens, np.int32)
    T, H = x.shape
    E = logits.shape[1]
    I = w2c.shape[2] * 2
    n = tok.size
    o = dict(idx=np.empty((n, k), np.int32), gates=np.empty((n, k), np.float64),
             xq=np.empty((n, H), np.int8), sx=np.empty(n, np.float32),
             hq=np.empty((n * k, I), np.int8), sh=np.empty(n * k, np.float32),
             y=np.empty((n, H), np.uint16))
    rc = _L().orc_forward_tokens(T, H, I, E, k, _p(x), _p(logits), _p(w1c), _p(w1s), _p(w2c),
                                 _p(w2s), _p(tok), n, _p(o["idx"]), _p(o["gates"]), _p(o["xq"]),
                                 _p(o["sx"]), _p(o["hq"]), _p(o["sh"]), _p(o["y"]), nthreads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return o


def forward_dense(x, logits, w1_codes, w1_scales, w2_codes, w2_scales, k: int):
    """Brute force: every token through every expert, dense gate mask."""
    x = _c(x, np.uint16)
    logits = _c(logits, np.float32)
    w1c, w1s, w2c, w2s = (_c(a, np.uint8) for a in (w1_codes, w1_scales, w2_codes, w2_scales))
    T, H = x.shape
    E = logits.shape[1]
    I = w2c.shape[2] * 2
    y64 = np.empty((T, H), np.float64)
    y = np.empty((T, H), np.uint16)
    rc = _L().orc_forward_dense(T, H, I, E, k, _p(x), _p(logits), _p(w1c), _p(w1s), _p(w2c),
                                _p(w2s), _p(y64), _p(y), nthreads())
    if rc != 0:
        raise ValueError("oracle rejected the arguments")
    return y64, y


# ---- FP8 block-quantised dense projection (fp8_oracle.cpp) ---------------------

def e4m3(code: int) -> float:
    """Value of an OCP E4M3 code (NaN for 0x7F / 0xFF)."""
    return _L().orc_e4m3(code)


def e4m3_code(v: float) -> int:
    """Nearest E4M3 code of v (|v| <= 448), ties to even."""
    return int(_L().orc_e4m3_code(v))


def fp8_quant_act(x_bits: np.ndarray):
    """x raw bf16 bits [T, K] -> (q [T, K] E4M3 codes, s [T, K/128] UE8M0 bytes)."""
    x = _c(x_bits, np.uint16)
    T, K = x.shape
    assert K % 128 == 0
    q = np.empty((T, K), np.uint8)
    s = np.empty((T, K // 128), np.uint8)
    _L().orc_fp8_quant_act(_p(x), T, K, _p(q), _p(s), nthreads())
    return q, s


def fp8_linear(q: np.ndarray, s: np.ndarray, wq: np.ndarray, ws: np.ndarray, want_f64: bool = False):
    """y[t, n] = bf16(sum_k dequant(q)[t,k] * dequant(wq)[n,k]); with want_f64 also
    the fp64 sums and the sums of |terms|."""
    q, s, wq, ws = _c(q, np.uint8), _c(s, np.uint8), _c(wq, np.uint8), _c(ws, np.uint8)
    T, K = q.shape
    N = wq.shape[0]
    assert wq.shape[1] == K and s.shape == (T, K // 128) and ws.shape == (N // 128, K // 128)
    y = np.empty((T, N), np.uint16)
    y64 = np.empty((T, N), np.float64) if want_f64 else None
    yabs = np.empty((T, N), np.float64) if want_f64 else None
    _L().orc_fp8_linear(_p(q), _p(s), _p(wq), _p(ws), T, N, K, _p(y), _p(y64), _p(yabs), nthreads())
    return (y, y64, yabs) if want_f64 else y
