"""Pins of the FP8 block-quantised projection oracle (oracle/fp8_oracle.cpp)
to sources other than itself; no GPU needed.

The pages name the format only ("FP8 dense projections", "FP8 block
quantization": "DeepSeek-V4-Flash on AMD gfx90a" abstract; "DeepSeek V4 Flash
on 8x R9600D" model facts).  The oracle's readings: OCP E4M3 codes, UE8M0
power-of-two scales per 128 x 128 weight block and per token x 128-input
activation block, the activation scale the smallest power of two that keeps
every code finite, codes by round-to-nearest-even, the product summed in fp64
and rounded once to bf16.  Each pin below would fail on a plausible slip: a
wrong exponent bias or subnormal rule (decode vs ml_dtypes), a wrong tie rule
(encode vs ml_dtypes' RNE cast), a scale one binade off (brute force on the
definition), a transposed or mis-indexed block scale (float64 matmul of the
dequantised operands, one block at a time).
"""
import ml_dtypes
import numpy as np
import pytest

import oracle
import synth


def test_e4m3_decode_matches_ml_dtypes():
    ref = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    got = np.array([oracle.e4m3(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got)) and nan.sum() == 2
    assert np.array_equal(ref[~nan], got[~nan])
    assert oracle.e4m3(0x7E) == 448.0 and oracle.e4m3(1) == 2.0 ** -9


def test_e4m3_encode_is_ml_dtypes_rne_cast():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-448, 448, 4000), rng.normal(0, 1e-2, 2000), rng.normal(0, 0.5, 2000)])
    mags = np.arange(0x7F, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mid = (mags[:-1] + mags[1:]) / 2      # every tie between neighbouring codes
    v = np.concatenate([v, mid, -mid, [0.0, 448.0, -448.0]])
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = np.array([oracle.e4m3_code(float(a)) for a in v], np.uint8)
    # -0.0 and +0.0: ml_dtypes keeps the sign of zero; so does the oracle
    assert np.array_equal(ref, got), np.nonzero(ref != got)[0][:5]


def _dequant_act(q, s):
    T, K = q.shape
    vals = q.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return vals * np.repeat(np.ldexp(1.0, s.astype(np.int64) - 127), 128, axis=1)


def test_quant_act_scale_rule_and_codes_by_definition():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(0, 1, (6, 512)), rng.normal(0, 1e-3, (2, 512)),
                        rng.uniform(-3e4, 3e4, (2, 512))]).astype(np.float32)
    x[3, 128:256] = 0.0                   # an all-zero block
    x[4, 0:128] = 448.0                   # amax exactly 448 * 2^0
    x[5, 256:384] = np.float32(448.0 * 2 ** -3) * np.sign(rng.normal(size=128))
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)          # truncate to bf16
    xb = synth.bf16_to_f32(bits).astype(np.float64)
    q, s = oracle.fp8_quant_act(bits)
    for t in range(x.shape[0]):
        for g in range(4):
            blk = xb[t, 128 * g:128 * (g + 1)]
            a = np.abs(blk).max()
            if a == 0:
                assert s[t, g] == 0 and not q[t, 128 * g:128 * (g + 1)].any()
                continue
            e = int(s[t, g]) - 127
            assert a <= 448.0 * 2.0 ** e and a > 448.0 * 2.0 ** (e - 1)   # smallest such power
            ref = (blk * 2.0 ** -e).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
            assert np.array_equal(q[t, 128 * g:128 * (g + 1)], ref)
    assert s[4, 0] == 127 and s[5, 2] == 124


def test_linear_equals_float64_matmul_of_dequantised_operands():
    rng = np.random.default_rng(2)
    T, N, K = 5, 256, 384
    x = rng.normal(0, 1, (T, K)).astype(np.float32)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    q, s = oracle.fp8_quant_act(bits)
    wq = rng.integers(0, 256, (N, K)).astype(np.uint8)
    wq[(wq & 0x7F) == 0x7F] = 0x3C          # no NaN codes
    ws = rng.integers(118, 124, (N // 128, K // 128)).astype(np.uint8)
    y, y64, yabs = oracle.fp8_linear(q, s, wq, ws, want_f64=True)
    wv = wq.view(ml_dtypes.float8_e4m3fn).astype(np.float64) * np.repeat(
        np.repeat(np.ldexp(1.0, ws.astype(np.int64) - 127), 128, axis=0), 128, axis=1)
    ref = _dequant_act(q, s) @ wv.T
    assert np.allclose(y64, ref, rtol=1e-13, atol=1e-13 * yabs.max())
    assert np.all(yabs >= np.abs(y64))
    # the output is the nearest bf16 of the fp64 sum
    yb = synth.bf16_to_f32(y).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 7)
    assert np.all(np.abs(yb - ref) <= 0.5 * ulp * (1 + 1e-9))


def test_linear_integer_special_case():
    # codes of small integers with unit scales (byte 127): an int64 matmul
    rng = np.random.default_rng(3)
    T, N, K = 3, 128, 256
    ints = np.array([0, 1, 2, 3, 4, -1, -2, -3, -4])
    codes = np.array([oracle.e4m3_code(float(v)) for v in ints], np.uint8)
    xi = rng.integers(0, len(ints), (T, K))
    wi = rng.integers(0, len(ints), (N, K))
    q, w = codes[xi], codes[wi]
    s = np.full((T, K // 128), 127, np.uint8)
    ws = np.full((N // 128, K // 128), 127, np.uint8)
    y, y64, _ = oracle.fp8_linear(q, s, w, ws, want_f64=True)
    assert np.array_equal(y64, (ints[xi].astype(np.int64) @ ints[wi].T.astype(np.int64)).astype(np.float64))
