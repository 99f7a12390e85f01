"""The fused front of moe_layer_forward (route, sort, x quant and plan in one
launch) against the CPU oracle and against the separate calls.

moe_layer_forward takes the fused launch when 0 < T < MOE_OPT_TC_MIN_ROWS and
T*k <= 1024 (every expert on the streaming GEMM).  Bit-exact: routing indices,
sort tables, INT8 codes and scales; gates to 1e-6 relative and y to the
layer's tolerance against the oracle.  Against moe_route + moe_sort +
moe_forward (the unfused launches on the same GEMM path) every table and y
must be bit-identical.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.test_gpu_parity import effective_tc_threshold

pytestmark = pytest.mark.gpu

Y_MAX_REL = 2e-2
Y_FRO_REL = 5e-3
GATE_REL = 1e-6


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _inputs(moe, d):
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                  cu(d["w2_scales"]))
    return packed, cu(d["logits"]), cu(d["x"]).view(torch.bfloat16)


def _debug(T, H, I, k):
    return dict(xq=torch.empty((T, H), dtype=torch.int8, device="cuda"),
                sx=torch.empty(T, dtype=torch.float32, device="cuda"),
                hq=torch.empty((T * k, I), dtype=torch.int8, device="cuda"),
                sh=torch.empty(T * k, dtype=torch.float32, device="cuda"))


def _layer(moe, w, packed, logits, x):
    """moe_layer_forward with debug dumps; returns tables, dumps, y, launches."""
    T, H, I, E, k = w.T, w.H, w.I, w.E, w.k
    ws = torch.full((moe.moe_layer_workspace_bytes(T, H, I, E, k),), 0xA5, dtype=torch.uint8, device="cuda")
    dbg = _debug(T, H, I, k)
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    n0 = moe.moe_launch_count()
    moe.moe_layer_forward(logits, x, packed, H, I, E, k, ws=ws, y=y, dbg=moe.make_debug(dbg))
    launches = moe.moe_launch_count() - n0
    torch.cuda.synchronize()
    assert moe.moe_check_device_flag(ws) == 0
    tabs = {n: t.clone() for n, t in moe.moe_layer_tables(ws, T, H, I, E, k).items()}
    return tabs, dbg, y, launches


FRONT_CASES = [
    ("tiny_T4", None),
    ("decode_T8", None),
    ("t1_e1", (1, 128, 1, 1, 128, 61)),      # one token, one expert
    ("ragged", (13, 384, 9, 3, 256, 62)),    # 39 pairs, ragged groups
    ("k_eq_e", (9, 256, 16, 16, 128, 63)),   # k = E = 16: every expert, the 16-slot route
    ("wide_e", (31, 128, 1024, 16, 128, 64)),  # E = 1024 (32 logits per lane), 496 pairs
]


def _case(name, shape):
    if shape is None:
        w = synth.WORKLOADS[name]
    else:
        w = synth.custom(name, *shape)
    return w, synth.make(w)


@pytest.mark.parametrize("name,shape", FRONT_CASES, ids=[c[0] for c in FRONT_CASES])
def test_fused_front_matches_oracle(moe, name, shape):
    w, d = _case(name, shape)
    assert w.T < effective_tc_threshold(moe, w.T) and w.T * w.k <= 1024
    packed, logits, x = _inputs(moe, d)
    tabs, dbg, y, launches = _layer(moe, w, packed, logits, x)
    # one fused launch + W1, SwiGLU/h quant, W2, combine
    assert launches == 5, launches
    o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"], d["w2_scales"],
                       w.k)
    assert np.array_equal(tabs["idx"].cpu().numpy(), o["idx"])
    g = tabs["gates"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - o["gates"]) <= GATE_REL * np.abs(o["gates"]))
    assert np.array_equal(tabs["perm"].cpu().numpy(), o["perm"])
    assert np.array_equal(tabs["pos"].cpu().numpy(), o["pos"])
    assert np.array_equal(tabs["offsets"].cpu().numpy(), o["offsets"])
    assert np.array_equal(dbg["xq"].cpu().numpy(), o["xq"])
    assert np.array_equal(dbg["sx"].cpu().numpy(), o["sx"])
    perm = o["perm"]
    assert np.array_equal(dbg["hq"].cpu().numpy(), o["hq"][perm])
    assert np.array_equal(dbg["sh"].cpu().numpy(), o["sh"][perm])
    yg = y.float().cpu().numpy().astype(np.float64)
    yo = synth.bf16_to_f32(o["y"]).astype(np.float64)
    m = np.abs(yo).max()
    assert np.abs(yg - yo).max() <= Y_MAX_REL * m
    assert np.linalg.norm(yg - yo) / max(np.linalg.norm(yo), 1e-300) <= Y_FRO_REL


@pytest.mark.parametrize("name,shape", FRONT_CASES, ids=[c[0] for c in FRONT_CASES])
def test_fused_front_bit_identical_to_separate_calls(moe, name, shape):
    w, d = _case(name, shape)
    T, H, I, E, k = w.T, w.H, w.I, w.E, w.k
    packed, logits, x = _inputs(moe, d)
    tabs, dbg, y, _ = _layer(moe, w, packed, logits, x)
    idx, gates = moe.moe_route(logits, k)
    perm, pos, offsets = moe.moe_sort(idx, E)
    dbg2 = _debug(T, H, I, k)
    y2 = moe.moe_forward(x, idx, gates, perm, pos, offsets, packed, H, I, E, debug=dbg2)
    torch.cuda.synchronize()
    assert torch.equal(tabs["idx"], idx)
    assert torch.equal(tabs["gates"].view(torch.int32), gates.view(torch.int32))
    assert torch.equal(tabs["perm"], perm)
    assert torch.equal(tabs["pos"], pos)
    assert torch.equal(tabs["offsets"], offsets)
    for n in ("xq", "hq"):
        assert torch.equal(dbg[n], dbg2[n]), n
    for n in ("sx", "sh"):
        assert torch.equal(dbg[n].view(torch.int32), dbg2[n].view(torch.int32)), n
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_layer_beyond_one_sort_chunk_takes_separate_launches(moe):
    # T below a raised tensor-core threshold but T*k = 1600 pairs > 1024: the
    # layer runs route, sort (two chunks), x quant and plan as their own kernels
    w = synth.custom("chunks", 100, 128, 32, 16, 128, 65)
    d = synth.make(w)
    old = moe.moe_get_option(moe.MOE_OPT_TC_MIN_ROWS)
    moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, 128)
    try:
        packed, logits, x = _inputs(moe, d)
        tabs, dbg, y, launches = _layer(moe, w, packed, logits, x)
    finally:
        moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, old)
    # route, sort count + scatter, x quant, plan, W1, h quant, W2, combine
    assert launches == 9, launches
    o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"], d["w2_scales"],
                       w.k)
    assert np.array_equal(tabs["perm"].cpu().numpy(), o["perm"])
    assert np.array_equal(tabs["offsets"].cpu().numpy(), o["offsets"])
    assert np.array_equal(dbg["hq"].cpu().numpy(), o["hq"][o["perm"]])
    yg = y.float().cpu().numpy().astype(np.float64)
    yo = synth.bf16_to_f32(o["y"]).astype(np.float64)
    assert np.abs(yg - yo).max() <= Y_MAX_REL * np.abs(yo).max()


def test_fused_front_layout_mismatch_flag(moe):
    # weights packed for E=4 used as E=2 through the fused front: FLAG_LAYOUT,
    # and the GEMMs stay out of the packed buffer
    w = synth.custom("m", 2, 128, 4, 2, 128, 66)
    d = synth.make(w)
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                  cu(d["w2_scales"]))
    logits = cu(d["logits"][:, :2].copy())
    x = cu(d["x"]).view(torch.bfloat16)
    ws = torch.empty(moe.moe_layer_workspace_bytes(2, 128, 128, 2, 2), dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward(logits, x, packed, 128, 128, 2, 2, ws=ws)
    assert moe.moe_check_device_flag(ws) & moe.FLAG_LAYOUT
