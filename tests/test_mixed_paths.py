"""Calls in which both grouped GEMMs run: experts with at least
MOE_OPT_TC_MIN_ROWS rows (default 32) on the tensor-core GEMM and the others on
the streaming GEMM, in one layer call, compared whole with the oracle.

In such a call the planner gives plane rows to tensor-core rows only, the
requant kernel takes h from two sources (the tensor-core epilogue's fp32 h, or
the streaming GEMM's fp64 sums) and the combine sums fp32 and fp64-derived Y
rows inside one token.  Bit-exact: idx, perm, pos, offsets, xq, sx, hq, sh;
y within max|dy| <= 2e-2 max|y_oracle| and relative Frobenius error <= 5e-3.
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from tests.test_gpu_parity import _check_layer  # noqa: E402


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


@pytest.fixture
def options(moe):
    """Set options for one test; the previous values come back afterwards."""
    keys = [moe.MOE_OPT_TC_MIN_ROWS, moe.MOE_OPT_TC_PAIR]
    old = {k_: moe.moe_get_option(k_) for k_ in keys}

    def set_(**kw):
        if "tc_min" in kw:
            moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, kw["tc_min"])
        if "pair" in kw:
            moe.moe_set_option(moe.MOE_OPT_TC_PAIR, kw["pair"])

    yield set_
    for k_, v in old.items():
        moe.moe_set_option(k_, v)


def _orc(d, k):
    return oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                          d["w2_scales"], k)


def _kinds(o, E, tc_min):
    counts = np.diff(o["offsets"])
    return int(((counts > 0) & (counts < tc_min)).sum()), int((counts >= tc_min).sum())


@pytest.mark.parametrize("pair", [0, 1])
def test_mixed_default_threshold(moe, options, pair):
    # bias c = 0.8 over 8 experts: rows per expert 274, 168, 76, 39 (tensor
    # cores) and 18, 15, 7, 3 (streaming) at the default threshold of 32
    options(tc_min=32, pair=pair)
    w = synth.custom("mix", 300, 512, 8, 2, 256, 81, 0.8)
    d = synth.make(w)
    o = _orc(d, w.k)
    n_stream, n_tc = _kinds(o, w.E, 32)
    assert n_stream >= 3 and n_tc >= 3, (n_stream, n_tc)
    _check_layer(moe, d, w, o)


@pytest.mark.parametrize("tc_min", [2, 40, 100])
def test_mixed_other_thresholds(moe, options, tc_min):
    # the same call with the split moved: 2 (all but the 1-row experts on
    # tensor cores), 40 and 100
    options(tc_min=tc_min)
    w = synth.custom("mix2", 257, 256, 16, 4, 384, 82, 1.0)
    d = synth.make(w)
    o = _orc(d, w.k)
    n_stream, n_tc = _kinds(o, w.E, tc_min)
    assert n_tc >= 1 and n_stream >= 1, (n_stream, n_tc)
    _check_layer(moe, d, w, o)


def _crafted(T, H, E, k, I, seed, top):
    """Inputs with hand-set logits: token t's j-th choice is expert top(t)[j]
    (logit 10 - j), every other expert gets logit -10."""
    w = synth.custom("craft", T, H, E, k, I, seed)
    d = synth.make(w)
    lg = np.full((T, E), -10.0, np.float32)
    for t in range(T):
        for j, e in enumerate(top(t)):
            lg[t, e] = 10.0 - j
    d["logits"] = lg
    return w, d


def test_threshold_edges_and_zero_row(moe, options):
    # experts with exactly 31 and 32 rows on both sides of the default
    # threshold, and an all-zero token (s = 0 end to end: codes, scales and its
    # output row are 0) landing in both kinds of expert
    options(tc_min=32)
    T = 63
    w, d = _crafted(T, 256, 4, 2, 128, 91, lambda t: (0 if t < 31 else 1, 2 if t % 2 == 0 else 3))
    d["x"][5] = 0        # -> experts 0 (31 rows, streaming) and 3 (31 rows, streaming)
    d["x"][40] = 0       # -> experts 1 (32 rows, tensor cores) and 2 (32 rows, tensor cores)
    o = _orc(d, w.k)
    assert list(np.diff(o["offsets"])) == [31, 32, 32, 31]
    assert o["sx"][5] == 0 and o["sx"][40] == 0
    _check_layer(moe, d, w, o)


def test_single_row_tensor_core_experts_among_streaming(moe, options):
    # tc_min = 1 with k = 1: every expert on tensor cores, most with 1-3 rows
    # (the smallest MMA, N = 16, padded rows ignored)
    options(tc_min=1)
    w = synth.custom("ones", 20, 256, 16, 1, 128, 92)
    d = synth.make(w)
    _check_layer(moe, d, w, _orc(d, w.k))
