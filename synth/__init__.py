"""Seeded synthetic inputs for the routed FP4 mixture-of-experts layer.

Random numbers and input preparation only: nothing in this package performs
the layer's arithmetic.  Both the CUDA library and the CPU oracle take their
inputs from here.  The generator (SplitMix64, counter-based) and the value
distributions are described in ``synth.c``.

Workloads follow the routed-MoE layer of DeepSeek-V4-Flash-style inference
(256 routed experts, 6 active per token; "DeepSeek V4 Flash on 8x R9600D"
blog post, model facts paragraph).  Sizes and distributions:

* x ~ N(0,1) -> fp32 -> bf16 (round to nearest even), shape [T, H]
* router weight W_r ~ 0.02 * N(0,1) in fp32, shape [E, H]
* W1 [E, 2I, H] and W2 [E, H, I] in canonical MXFP4: E2M1 codes uniform over
  the 16 nibbles (two per byte, even element in the low nibble) and one UE8M0
  scale byte per 32 consecutive input-dimension elements, uniform in
  {120, ..., 124}
* router logits = fp32(sum_h x[t,h] * W_r[e,h] + b_e), summed in fp64; the
  skewed prefill workloads add b_e = c * ln(1 / (e + 1)) with c = 3 (as
  specified) and c = 1.25 (a labelled variant whose expert counts match the
  described "about 40 experts receive 0 tokens" more closely).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "libmoe_synth.so")

TID_X, TID_WR, TID_W1C, TID_W1S, TID_W2C, TID_W2S = range(6)
SCALE_BASE, SCALE_SPAN = 120, 5


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    seed: int
    bias_coef: float = 0.0

    @property
    def P(self) -> int:
        return self.T * self.k


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_T4", 4, 256, 16, 2, 128, 0),
        Workload("decode_T8", 8, 4096, 256, 6, 2048, 1),
        Workload("decode_T64", 64, 4096, 256, 6, 2048, 2),
        Workload("prefill_T4604", 4604, 4096, 256, 6, 2048, 3),
        Workload("prefill_skew_T16384", 16384, 4096, 256, 6, 2048, 4, 3.0),
        # the same tokens with a milder bias (c = 1.25): 29 empty experts, the
        # top expert takes 14,793 rows, 150 experts get 1-31 rows -- load
        # balance, empty groups and both GEMM kernels in one call
        Workload("prefill_skew1.25_T16384", 16384, 4096, 256, 6, 2048, 4, 1.25),
    ]
}


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``_build/libmoe_synth.so`` (gcc, no fast-math)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-ffp-contract=off",
             "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        u64, u32, i64, i32, vp = (ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int64, ctypes.c_int,
                                  ctypes.c_void_p)
        _lib.synth_normals_f32.argtypes = [u64, u32, ctypes.c_float, vp, i64, i32]
        _lib.synth_normals_bf16.argtypes = [u64, u32, vp, i64, i32]
        _lib.synth_bytes.argtypes = [u64, u32, vp, i64, i32]
        _lib.synth_uniform_bytes.argtypes = [u64, u32, u32, u32, vp, i64, i32]
        _lib.synth_router_logits.argtypes = [vp, vp, vp, i32, i32, i32, vp, i32]
        _lib.synth_u64.argtypes = [u64, u32, u64]
        _lib.synth_u64.restype = u64
        _lib.synth_splitmix64_at.argtypes = [u64, u64]
        _lib.synth_splitmix64_at.restype = u64
    return _lib


def _nt() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def splitmix64_at(state: int, i: int) -> int:
    """Output number i of a plain SplitMix64 generator started in `state`."""
    return int(_L().synth_splitmix64_at(state, i))


def u64_at(seed: int, tid: int, i: int) -> int:
    """Output number i of tensor stream `tid` (for generator pins)."""
    return int(_L().synth_u64(seed, tid, i))


def normals_f32(seed: int, tid: int, n: int, scale: float = 1.0) -> np.ndarray:
    out = np.empty(n, np.float32)
    _L().synth_normals_f32(seed, tid, scale, _ptr(out), n, _nt())
    return out


def x_bf16(seed: int, T: int, H: int) -> np.ndarray:
    """Activations as raw bf16 bits (uint16), shape [T, H]."""
    out = np.empty((T, H), np.uint16)
    _L().synth_normals_bf16(seed, TID_X, _ptr(out), T * H, _nt())
    return out


def router_weight(seed: int, E: int, H: int) -> np.ndarray:
    return normals_f32(seed, TID_WR, E * H, 0.02).reshape(E, H)


def code_bytes(seed: int, tid: int, shape) -> np.ndarray:
    out = np.empty(shape, np.uint8)
    _L().synth_bytes(seed, tid, _ptr(out), out.size, _nt())
    return out


def scale_bytes(seed: int, tid: int, shape, base: int = SCALE_BASE, span: int = SCALE_SPAN) -> np.ndarray:
    out = np.empty(shape, np.uint8)
    _L().synth_uniform_bytes(seed, tid, base, span, _ptr(out), out.size, _nt())
    return out


def router_bias(E: int, coef: float) -> np.ndarray | None:
    if coef == 0.0:
        return None
    return np.array([coef * math.log(1.0 / (e + 1)) for e in range(E)], np.float64)


def router_logits(x: np.ndarray, wr: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, np.float64)
    _L().synth_router_logits(_ptr(np.ascontiguousarray(x)), _ptr(np.ascontiguousarray(wr)),
                             None if b is None else _ptr(b), T, H, E, _ptr(out), _nt())
    return out


def weights(w: Workload, scale_base: int = SCALE_BASE, scale_span: int = SCALE_SPAN) -> dict:
    """Canonical MXFP4 expert weights of a workload.

    w1_codes [E, 2I, H/2], w1_scales [E, 2I, H/32], w2_codes [E, H, I/2],
    w2_scales [E, H, I/32], all uint8.  W1 rows [0, I) are gate, [I, 2I) up.
    """
    E, H, I = w.E, w.H, w.I
    return dict(
        w1_codes=code_bytes(w.seed, TID_W1C, (E, 2 * I, H // 2)),
        w1_scales=scale_bytes(w.seed, TID_W1S, (E, 2 * I, H // 32), scale_base, scale_span),
        w2_codes=code_bytes(w.seed, TID_W2C, (E, H, I // 2)),
        w2_scales=scale_bytes(w.seed, TID_W2S, (E, H, I // 32), scale_base, scale_span),
    )


def activations(w: Workload, T: int | None = None) -> dict:
    """x (bf16 bits [T,H]) and router logits (fp32 [T,E]) of a workload."""
    T = w.T if T is None else T
    x = x_bf16(w.seed, T, w.H)
    wr = router_weight(w.seed, w.E, w.H)
    return dict(x=x, logits=router_logits(x, wr, router_bias(w.E, w.bias_coef)))


def make(w: Workload) -> dict:
    d = activations(w)
    d.update(weights(w))
    return d


def custom(name: str, T: int, H: int, E: int, k: int, I: int, seed: int, bias_coef: float = 0.0) -> Workload:
    return Workload(name, T, H, E, k, I, seed, bias_coef)


# ---- FP8 block-quantised dense projection inputs --------------------------------
# x [T, K] ~ N(0, 1) in bf16 (the activation generator above); weights as
# uniform E4M3 code bytes (the two NaN bytes 0x7F / 0xFF replaced by their
# neighbours 0x7E / 0xFE, 448 and -448) and one UE8M0 scale byte per 128 x 128
# block, uniform in {118, ..., 122}.  Shapes use the layer's hidden size.
TID_F8W, TID_F8S = 16, 17


@dataclass(frozen=True)
class DenseWorkload:
    name: str
    T: int
    N: int
    K: int
    seed: int


DENSE_WORKLOADS = {
    w.name: w
    for w in [
        DenseWorkload("dense_T8", 8, 4096, 4096, 11),
        DenseWorkload("dense_T4604", 4604, 4096, 4096, 13),
    ]
}


def fp8_weights(seed: int, N: int, K: int) -> dict:
    codes = code_bytes(seed, TID_F8W, (N, K))
    nan = (codes & 0x7F) == 0x7F
    codes[nan] -= 1
    scales = scale_bytes(seed, TID_F8S, (N // 128, K // 128), 118, 5)
    return dict(w_codes=codes, w_scales=scales)


def make_dense(w: DenseWorkload) -> dict:
    d = dict(x=x_bf16(w.seed, w.T, w.K))
    d.update(fp8_weights(w.seed, w.N, w.K))
    return d


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Raw bf16 bits (uint16) -> float32 values (exact widening)."""
    return (a.astype(np.uint32) << 16).view(np.float32)
