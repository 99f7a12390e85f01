"""ctypes binding of libmoe.so (include/moe.h), argument marshalling only.

Every function takes torch CUDA tensors, passes their data pointers and the
current CUDA stream to the C ABI, and raises MoeError on a non-zero status.
All arithmetic happens in the library's CUDA kernels; there is no fallback:
importing this module without the built library raises ImportError.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmoe.so")

MOE_OK = 0
STATUS = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED_SHAPE",
          -3: "MOE_ERR_CUDA", -4: "MOE_ERR_LAYOUT_MISMATCH", -5: "MOE_ERR_TIMEOUT",
          -6: "MOE_ERR_DEVICE_FLAG"}
FLAG_BAD_EXPERT, FLAG_BAD_SCALE, FLAG_LAYOUT, FLAG_TIMEOUT, FLAG_BOUNDS = 1, 2, 4, 8, 16

# Exported symbols of include/moe.h, in declaration order.
SYMBOLS = ["moe_last_error", "moe_packed_bytes", "moe_pack_weights", "moe_unpack_weights",
           "moe_router_logits", "moe_route", "moe_sort_workspace_bytes", "moe_sort", "moe_sort_static", "moe_workspace_bytes",
           "moe_forward", "moe_layer_workspace_bytes", "moe_layer_forward", "moe_layer_router_workspace_bytes",
           "moe_layer_forward_with_router", "moe_layer_tables",
           "moe_quant_rows_f32", "moe_exp_f32", "moe_swiglu_f32",
           "moe_fp8_packed_bytes", "moe_fp8_pack_weights", "moe_fp8_unpack_weights", "moe_fp8_workspace_bytes",
           "moe_fp8_linear",
           "moe_set_option", "moe_get_option", "moe_launch_count", "moe_check_device_flag"]


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class moe_dims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("H", ctypes.c_int), ("I", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int)]


class moe_debug(ctypes.Structure):
    _fields_ = [("xq", ctypes.c_void_p), ("sx", ctypes.c_void_p), ("hq", ctypes.c_void_p),
                ("sh", ctypes.c_void_p), ("events", ctypes.c_void_p * 4)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python fp4_routed_mixture_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    D = ctypes.POINTER(moe_dims)
    sig = {
        "moe_last_error": ([ctypes.c_char_p, sz], sz),
        "moe_packed_bytes": ([D], sz),
        "moe_pack_weights": ([D, vp, vp, vp, vp, vp, vp], i32),
        "moe_unpack_weights": ([D, vp, vp, vp, vp, vp, vp], i32),
        "moe_router_logits": ([vp, vp, vp, i32, i32, i32, vp, vp], i32),
        "moe_route": ([vp, i32, i32, i32, vp, vp, vp], i32),
        "moe_sort_workspace_bytes": ([i32, i32, i32], sz),
        "moe_sort": ([vp, i32, i32, i32, vp, vp, vp, vp, sz, vp], i32),
        "moe_sort_static": ([vp, i32, i32, i32, vp, vp, vp, vp], i32),
        "moe_workspace_bytes": ([D, i32], sz),
        "moe_forward": ([D, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, ctypes.POINTER(moe_debug), vp], i32),
        "moe_layer_workspace_bytes": ([D, i32], sz),
        "moe_layer_forward": ([D, vp, vp, vp, vp, vp, sz, ctypes.POINTER(moe_debug), vp], i32),
        "moe_layer_router_workspace_bytes": ([D, i32], sz),
        "moe_layer_forward_with_router": ([D, vp, vp, vp, vp, vp, vp, sz, ctypes.POINTER(moe_debug), vp], i32),
        "moe_layer_tables": ([D, vp] + [ctypes.POINTER(vp)] * 5, i32),
        "moe_quant_rows_f32": ([vp, i32, i32, vp, vp, vp], i32),
        "moe_exp_f32": ([vp, vp, ctypes.c_int64, vp], i32),
        "moe_swiglu_f32": ([vp, vp, vp, ctypes.c_int64, vp], i32),
        "moe_fp8_packed_bytes": ([i32, i32], sz),
        "moe_fp8_pack_weights": ([i32, i32, vp, vp, vp, vp], i32),
        "moe_fp8_unpack_weights": ([i32, i32, vp, vp, vp, vp], i32),
        "moe_fp8_workspace_bytes": ([i32, i32, i32], sz),
        "moe_fp8_linear": ([vp, i32, i32, i32, vp, vp, vp, sz, vp, vp, vp], i32),
        "moe_set_option": ([i32, i32], i32),
        "moe_get_option": ([i32], i32),
        "moe_launch_count": ([], ctypes.c_ulonglong),
        "moe_check_device_flag": ([vp, ctypes.POINTER(ctypes.c_int32), vp], i32),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes, f.restype = args, res
    return lib


lib = _load()


def last_error() -> str:
    buf = ctypes.create_string_buffer(1024)
    lib.moe_last_error(buf, 1024)
    return buf.value.decode()


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, last_error())


def _ptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "need a contiguous CUDA tensor"
    return t.data_ptr()


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dims(T, H, I, E, k):
    return moe_dims(T, H, I, E, k)


def _empty_aligned(nbytes: int, device) -> torch.Tensor:
    """Device buffer of nbytes (torch's allocator returns 256-byte aligned blocks)."""
    t = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t


# ---- sizes ----------------------------------------------------------------------------

def moe_packed_bytes(H: int, I: int, E: int) -> int:
    d = _dims(0, H, I, E, 1)
    n = lib.moe_packed_bytes(ctypes.byref(d))
    if n == 0:
        raise MoeError(-2, "unsupported dims")
    return n


def moe_workspace_bytes(T_max: int, H: int, I: int, E: int, k: int) -> int:
    d = _dims(T_max, H, I, E, k)
    n = lib.moe_workspace_bytes(ctypes.byref(d), T_max)
    if n == 0:
        raise MoeError(-2, "unsupported dims")
    return n


def moe_sort_workspace_bytes(T_max: int, k: int, E: int) -> int:
    return lib.moe_sort_workspace_bytes(T_max, k, E)


# ---- calls ------------------------------------------------------------------------------

def moe_pack_weights(w1_codes, w1_scales, w2_codes, w2_scales, stream=None) -> torch.Tensor:
    """Canonical MXFP4 (uint8 CUDA tensors [E,2I,H/2], [E,2I,H/32], [E,H,I/2],
    [E,H,I/32]) -> packed device layout (uint8 tensor).  Synchronises."""
    E, N1, Hh = w1_codes.shape
    H, I = 2 * Hh, N1 // 2
    packed = _empty_aligned(moe_packed_bytes(H, I, E), w1_codes.device)
    d = _dims(0, H, I, E, 1)
    _check(lib.moe_pack_weights(ctypes.byref(d), _ptr(w1_codes), _ptr(w1_scales), _ptr(w2_codes),
                                _ptr(w2_scales), _ptr(packed), _stream(stream)))
    return packed


def moe_unpack_weights(packed, H: int, I: int, E: int, stream=None):
    dev = packed.device
    w1c = torch.empty((E, 2 * I, H // 2), dtype=torch.uint8, device=dev)
    w1s = torch.empty((E, 2 * I, H // 32), dtype=torch.uint8, device=dev)
    w2c = torch.empty((E, H, I // 2), dtype=torch.uint8, device=dev)
    w2s = torch.empty((E, H, I // 32), dtype=torch.uint8, device=dev)
    d = _dims(0, H, I, E, 1)
    _check(lib.moe_unpack_weights(ctypes.byref(d), _ptr(packed), _ptr(w1c), _ptr(w1s), _ptr(w2c),
                                  _ptr(w2s), _stream(stream)))
    return w1c, w1s, w2c, w2s


def moe_router_logits(x, w_router, bias=None, out=None, stream=None):
    """x [T,H] bf16, w_router [E,H] fp32, bias [E] fp32 or None -> logits [T,E] fp32."""
    T, H = x.shape
    E = w_router.shape[0]
    if out is None:
        out = torch.empty((T, E), dtype=torch.float32, device=x.device)
    _check(lib.moe_router_logits(_ptr(x), _ptr(w_router), _ptr(bias), T, H, E, _ptr(out), _stream(stream)))
    return out


def moe_route(logits, k: int, out=None, stream=None):
    """logits [T,E] fp32 -> (topk_idx [T,k] int32, gates [T,k] fp32)."""
    T, E = logits.shape
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=logits.device),
               torch.empty((T, k), dtype=torch.float32, device=logits.device))
    idx, gates = out
    _check(lib.moe_route(_ptr(logits), T, E, k, _ptr(idx), _ptr(gates), _stream(stream)))
    return idx, gates


def moe_sort(topk_idx, E: int, ws=None, out=None, stream=None):
    """topk_idx [T,k] int32 -> (perm [P], pos [P], offsets [E+1]) int32."""
    T, k = topk_idx.shape
    dev = topk_idx.device
    if ws is None:
        ws = _empty_aligned(moe_sort_workspace_bytes(T, k, E), dev)
    if out is None:
        out = (torch.empty(T * k, dtype=torch.int32, device=dev),
               torch.empty(T * k, dtype=torch.int32, device=dev),
               torch.empty(E + 1, dtype=torch.int32, device=dev))
    perm, pos, offsets = out
    _check(lib.moe_sort(_ptr(topk_idx), T, k, E, _ptr(perm), _ptr(pos), _ptr(offsets), _ptr(ws),
                        ws.numel(), _stream(stream)))
    return perm, pos, offsets


def moe_sort_static(topk_idx, E: int, out=None, stream=None):
    """moe_sort using the library's own fixed scratch (no workspace argument);
    T*k <= 65536 and E <= 1024."""
    T, k = topk_idx.shape
    dev = topk_idx.device
    if out is None:
        out = (torch.empty(T * k, dtype=torch.int32, device=dev),
               torch.empty(T * k, dtype=torch.int32, device=dev),
               torch.empty(E + 1, dtype=torch.int32, device=dev))
    perm, pos, offsets = out
    _check(lib.moe_sort_static(_ptr(topk_idx), T, k, E, _ptr(perm), _ptr(pos), _ptr(offsets),
                               _stream(stream)))
    return perm, pos, offsets


def moe_forward(x, topk_idx, gates, perm, pos, offsets, packed, H: int, I: int, E: int,
                ws=None, y=None, debug: dict | None = None, stream=None):
    """x [T,H] bf16 -> y [T,H] bf16.  `debug` may hold CUDA tensors named xq,
    sx, hq, sh to receive the INT8 activations (hq/sh in sorted order)."""
    T = x.shape[0]
    k = topk_idx.shape[1]
    dev = x.device
    if ws is None:
        ws = _empty_aligned(moe_workspace_bytes(T, H, I, E, k), dev)
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    d = _dims(T, H, I, E, k)
    dbg = make_debug(debug) if debug else None
    _check(lib.moe_forward(ctypes.byref(d), _ptr(x), _ptr(topk_idx), _ptr(gates), _ptr(perm),
                           _ptr(pos), _ptr(offsets), _ptr(packed), _ptr(y), _ptr(ws), ws.numel(),
                           ctypes.byref(dbg) if dbg is not None else None, _stream(stream)))
    return y


def moe_layer_workspace_bytes(T_max: int, H: int, I: int, E: int, k: int) -> int:
    d = _dims(T_max, H, I, E, k)
    n = lib.moe_layer_workspace_bytes(ctypes.byref(d), T_max)
    if n == 0:
        raise MoeError(-2, "unsupported dims")
    return n


def make_debug(debug: dict | None = None, events=None):
    """moe_debug struct from optional dump tensors and up to 4 torch.cuda.Event
    objects (recorded once here so that their handles exist)."""
    dbg = moe_debug()
    for n in ("xq", "sx", "hq", "sh"):
        setattr(dbg, n, _ptr((debug or {}).get(n)))
    for j, ev in enumerate(events or []):
        if ev is not None:
            ev.record()
            dbg.events[j] = ev.cuda_event
    return dbg


def moe_layer_forward(logits, x, packed, H: int, I: int, E: int, k: int, ws=None, y=None,
                      dbg: moe_debug | None = None, stream=None):
    """The whole layer: logits [T,E] fp32, x [T,H] bf16 -> y [T,H] bf16."""
    T = x.shape[0]
    dev = x.device
    if ws is None:
        ws = _empty_aligned(moe_layer_workspace_bytes(T, H, I, E, k), dev)
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    d = _dims(T, H, I, E, k)
    _check(lib.moe_layer_forward(ctypes.byref(d), _ptr(logits), _ptr(x), _ptr(packed), _ptr(y),
                                 _ptr(ws), ws.numel(), ctypes.byref(dbg) if dbg is not None else None,
                                 _stream(stream)))
    return y


def moe_layer_router_workspace_bytes(T_max: int, H: int, I: int, E: int, k: int) -> int:
    d = _dims(T_max, H, I, E, k)
    n = lib.moe_layer_router_workspace_bytes(ctypes.byref(d), T_max)
    if n == 0:
        raise MoeError(-2, "unsupported dims")
    return n


def moe_layer_forward_with_router(x, w_router, bias, packed, H: int, I: int, E: int, k: int, ws=None, y=None,
                                  dbg: moe_debug | None = None, stream=None):
    """Router projection then the whole layer: x [T,H] bf16, w_router [E,H] fp32,
    bias [E] fp32 or None -> y [T,H] bf16."""
    T = x.shape[0]
    dev = x.device
    if ws is None:
        ws = _empty_aligned(moe_layer_router_workspace_bytes(T, H, I, E, k), dev)
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    d = _dims(T, H, I, E, k)
    _check(lib.moe_layer_forward_with_router(ctypes.byref(d), _ptr(x), _ptr(w_router), _ptr(bias), _ptr(packed),
                                             _ptr(y), _ptr(ws), ws.numel(),
                                             ctypes.byref(dbg) if dbg is not None else None, _stream(stream)))
    return y


def moe_layer_tables(ws, T: int, H: int, I: int, E: int, k: int):
    """Views of the routing tables moe_layer_forward left in `ws` (a uint8 CUDA
    tensor): topk_idx [T,k] int32, gates [T,k] fp32, perm [T*k], pos [T*k] and
    offsets [E+1] int32."""
    d = _dims(T, H, I, E, k)
    ptrs = [ctypes.c_void_p() for _ in range(5)]
    _check(lib.moe_layer_tables(ctypes.byref(d), _ptr(ws), *[ctypes.byref(p) for p in ptrs]))
    base = ws.data_ptr()

    def view(p, n, dtype, shape):
        off = p.value - base
        assert 0 <= off and off + 4 * n <= ws.numel()
        return ws[off:off + 4 * n].view(dtype).view(shape)

    P = T * k
    return dict(idx=view(ptrs[0], P, torch.int32, (T, k)), gates=view(ptrs[1], P, torch.float32, (T, k)),
                perm=view(ptrs[2], P, torch.int32, (P,)), pos=view(ptrs[3], P, torch.int32, (P,)),
                offsets=view(ptrs[4], E + 1, torch.int32, (E + 1,)))


def moe_quant_rows_f32(v, stream=None):
    rows, cols = v.shape
    q = torch.empty((rows, cols), dtype=torch.int8, device=v.device)
    s = torch.empty(rows, dtype=torch.float32, device=v.device)
    _check(lib.moe_quant_rows_f32(_ptr(v), rows, cols, _ptr(q), _ptr(s), _stream(stream)))
    return q, s


def moe_exp_f32(x, stream=None):
    y = torch.empty_like(x)
    _check(lib.moe_exp_f32(_ptr(x), _ptr(y), x.numel(), _stream(stream)))
    return y


def moe_swiglu_f32(g, u, stream=None):
    h = torch.empty_like(g)
    _check(lib.moe_swiglu_f32(_ptr(g), _ptr(u), _ptr(h), g.numel(), _stream(stream)))
    return h


def moe_fp8_pack_weights(w_codes, w_scales, stream=None) -> torch.Tensor:
    """FP8 weights, canonical uint8 CUDA tensors [N, K] (E4M3 codes) and
    [N/128, K/128] (UE8M0 bytes) -> packed device layout.  Synchronises."""
    N, K = w_codes.shape
    n = lib.moe_fp8_packed_bytes(N, K)
    if n == 0:
        raise MoeError(-2, "unsupported dims")
    packed = _empty_aligned(n, w_codes.device)
    _check(lib.moe_fp8_pack_weights(N, K, _ptr(w_codes), _ptr(w_scales), _ptr(packed), _stream(stream)))
    return packed


def moe_fp8_unpack_weights(packed, N: int, K: int, stream=None):
    wq = torch.empty((N, K), dtype=torch.uint8, device=packed.device)
    ws = torch.empty((N // 128, K // 128), dtype=torch.uint8, device=packed.device)
    _check(lib.moe_fp8_unpack_weights(N, K, _ptr(packed), _ptr(wq), _ptr(ws), _stream(stream)))
    return wq, ws


def moe_fp8_linear(x, packed, N: int, ws=None, y=None, debug: dict | None = None, stream=None):
    """x [T, K] bf16 -> y [T, N] bf16 through the FP8 packed weights.  `debug`
    may hold uint8 CUDA tensors q [T, K] and s [T, K/128] for the quantised x."""
    T, K = x.shape
    if ws is None:
        ws = _empty_aligned(lib.moe_fp8_workspace_bytes(T, N, K), x.device)
    if y is None:
        y = torch.empty((T, N), dtype=torch.bfloat16, device=x.device)
    dq = (debug or {}).get("q")
    ds = (debug or {}).get("s")
    _check(lib.moe_fp8_linear(_ptr(x), T, N, K, _ptr(packed), _ptr(y), _ptr(ws), ws.numel(), _ptr(dq), _ptr(ds),
                              _stream(stream)))
    return y


MOE_OPT_TC_MIN_ROWS = 1
MOE_OPT_TC_PAIR = 2
MOE_OPT_WAIT_LIMIT_US = 3
MOE_OPT_TEST_TIMEOUT = 4
MOE_OPT_TC_A_TMEM = 5
MOE_OPT_TC_FORM = 6


def moe_set_option(option: int, value: int):
    _check(lib.moe_set_option(option, value))


def moe_get_option(option: int) -> int:
    return int(lib.moe_get_option(option))


def moe_launch_count() -> int:
    return int(lib.moe_launch_count())


def moe_check_device_flag(ws, stream=None) -> int:
    """Device error word of a workspace (synchronises).  Returns the bits."""
    f = ctypes.c_int32(0)
    st = lib.moe_check_device_flag(_ptr(ws), ctypes.byref(f), _stream(stream))
    if st not in (MOE_OK, -6):
        _check(st)
    return f.value
