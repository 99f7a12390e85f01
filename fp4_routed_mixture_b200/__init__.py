"""B200 (sm_100a) routed FP4 mixture-of-experts layer.

The layer of DeepSeek-V4-Flash-style inference that "DeepSeek-V4-Flash on AMD
gfx90a: Correctness Recovery and Inference Performance Engineering" (abstract)
builds from packed FP4 expert weights, INT8 activations, expert sorting and
W1/W2 expert projections, with 256 routed experts and 6 active per token
("DeepSeek V4 Flash on 8x R9600D", model facts).

The computation lives in hand-written CUDA kernels behind the C ABI of
include/moe.h (libmoe.so); this package is the thin ctypes binding with the
same names.  Build the library with ``python fp4_routed_mixture_b200/build.py``.
"""
from .binding import (FLAG_BAD_EXPERT, FLAG_BAD_SCALE, FLAG_BOUNDS, FLAG_LAYOUT, FLAG_TIMEOUT,
                      LIB_PATH, SYMBOLS, MoeError, lib, moe_check_device_flag, moe_forward,
                      moe_pack_weights, moe_packed_bytes, moe_quant_rows_f32, moe_route, moe_router_logits, moe_sort,
                      moe_sort_workspace_bytes, moe_unpack_weights, moe_workspace_bytes,
                      moe_exp_f32, moe_swiglu_f32, moe_layer_forward, moe_layer_tables,
                      moe_layer_workspace_bytes, make_debug, moe_launch_count,
                      moe_set_option, moe_get_option, MOE_OPT_TC_MIN_ROWS, MOE_OPT_TC_PAIR,
                      MOE_OPT_WAIT_LIMIT_US, MOE_OPT_TEST_TIMEOUT, MOE_OPT_TC_A_TMEM,
                      MOE_OPT_TC_FORM,
                      moe_sort_static, moe_layer_forward_with_router, moe_layer_router_workspace_bytes,
                      moe_fp8_pack_weights, moe_fp8_unpack_weights, moe_fp8_linear)

__all__ = ["moe_layer_forward", "moe_layer_tables", "moe_layer_workspace_bytes", "make_debug", "moe_pack_weights", "moe_unpack_weights", "moe_router_logits", "moe_route", "moe_sort", "moe_forward",
           "moe_quant_rows_f32", "moe_exp_f32", "moe_swiglu_f32", "moe_check_device_flag", "moe_packed_bytes", "moe_workspace_bytes",
           "moe_sort_workspace_bytes", "MoeError", "LIB_PATH", "SYMBOLS", "lib"]
