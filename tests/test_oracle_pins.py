"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to an independent source: a library
routine (ml_dtypes' OCP MX decoders, libm exp, numpy's stable sort, scipy's
softmax, a float64 BLAS matmul, Python's round-half-even), a closed form, an
invariant, or a brute force.  The method itself is named by the paper
"DeepSeek-V4-Flash on AMD gfx90a: Correctness Recovery and Inference
Performance Engineering" (abstract): FP4 routed experts, INT8 activation
quantisation, expert sorting, W1/W2 expert projections.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import scipy.special

import oracle
import synth


# ---- generator known answers (SplitMix64, Steele/Lea/Flood 2014) --------------

def test_splitmix64_known_answers():
    assert synth.splitmix64_at(0, 0) == 0xE220A8397B1DCDAF
    assert [synth.splitmix64_at(1234567, i) for i in range(3)] == [
        6457827717110365317, 3203168211198807973, 9817491932198370423]


def test_generator_distributions():
    x = synth.bf16_to_f32(synth.x_bf16(7, 64, 4096)).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    s = synth.scale_bytes(7, synth.TID_W1S, (1 << 20,))
    assert s.min() == 120 and s.max() == 124
    cnt = np.bincount(s)[120:]
    assert np.all(np.abs(cnt / cnt.sum() - 0.2) < 0.005)
    c = synth.code_bytes(7, synth.TID_W1C, (1 << 20,))
    nib = np.concatenate([c & 15, c >> 4])
    assert np.all(np.abs(np.bincount(nib, minlength=16) / nib.size - 1 / 16) < 0.002)


# ---- FP4 / scale decode ---------------------------------------------------------

def test_e2m1_decode_matches_ml_dtypes():
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.array([oracle.e2m1(c) for c in range(16)])
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))  # code 8 is -0


def test_e8m0_decode_matches_ml_dtypes():
    s = np.arange(255, dtype=np.uint8)
    ref = s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    got = np.array([oracle.e8m0(int(v)) for v in s])
    assert np.array_equal(got, ref)


# ---- the layer's exp --------------------------------------------------------------

def _ulp_err(got32, ref64):
    got = got32.astype(np.float64)
    ulp = np.spacing(np.abs(ref64).astype(np.float32)).astype(np.float64)
    return np.abs(got - ref64) / ulp


def test_exp_within_2ulp_of_libm():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-87.3, 88.7, 1 << 20), rng.uniform(-1, 1, 1 << 18),
                        np.linspace(-87.3, 88.7, 100001)]).astype(np.float32)
    got = oracle.exp_f32(x)
    ref = np.exp(x.astype(np.float64))
    assert _ulp_err(got, ref).max() <= 2.0


def test_exp_special_values():
    big = oracle.exp_f32(np.float32([88.72283, 88.7229, 89.0, 100.0, np.inf]))
    assert np.isfinite(big[0]) and np.all(np.isinf(big[1:]))
    small = oracle.exp_f32(np.float32([-104.0, -103.9, -110.0, -np.inf]))
    assert np.all(small[2:] == 0.0)
    # subnormal range: within 1 subnormal step of the true value
    x = np.linspace(-103.9, -87.4, 5001).astype(np.float32)
    got = oracle.exp_f32(x).astype(np.float64)
    assert np.all(np.abs(got - np.exp(x.astype(np.float64))) <= 2 ** -149 * 1.01 + 3e-7 * got)
    assert np.isnan(oracle.exp_f32(np.float32([np.nan]))[0])
    assert oracle.exp_f32(np.float32([0.0]))[0] == 1.0


def test_swiglu_close_to_silu_times_up():
    rng = np.random.default_rng(1)
    g = rng.normal(0, 8, 20000).astype(np.float32)
    u = rng.normal(0, 8, 20000).astype(np.float32)
    got = np.array([oracle.swiglu(float(a), float(b)) for a, b in zip(g, u)])
    gd, ud = g.astype(np.float64), u.astype(np.float64)
    ref = gd * scipy.special.expit(gd) * ud
    assert np.all(np.abs(got - ref) <= 4e-7 * np.abs(ref) + 1e-30)
    # large negative g: exp overflows to inf and the product is a signed zero
    assert oracle.swiglu(-200.0, 3.0) == 0.0


# ---- quantisation -------------------------------------------------------------------

def test_quant_extremes_map_to_127():
    v = np.float32([[0.5, -3.25, 3.25, 1.0], [-7.0, 2.0, 0.0, 7.0]])
    q, s = oracle.quant_rows(v)
    assert q[0, 2] == 127 and q[0, 1] == -127 and q[1, 0] == -127 and q[1, 3] == 127
    assert s[0] == np.float32(3.25) / np.float32(127)


def test_quant_ties_round_half_even():
    # a = 127 makes s exactly 1, so q = round-half-even(v); Python's round() is half-even.
    vals = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 126.5, -126.5, 10.49, 10.51, 127.0]
    v = np.float32([vals])
    q, s = oracle.quant_rows(v)
    assert s[0] == 1.0
    assert list(q[0]) == [max(-127, min(127, round(x))) for x in vals]


def test_quant_zero_row():
    q, s = oracle.quant_rows(np.zeros((2, 64), np.float32))
    assert np.all(q == 0) and np.all(s == 0)


def test_quant_error_bound_random():
    rng = np.random.default_rng(2)
    v = rng.normal(0, 3, (64, 2048)).astype(np.float32)
    q, s = oracle.quant_rows(v)
    assert np.all(np.abs(q).max(axis=1) == 127)
    err = np.abs(v.astype(np.float64) - q.astype(np.float64) * s[:, None])
    assert np.all(err <= s[:, None] * (0.5 + 1e-5))


# ---- routing ------------------------------------------------------------------------

# ---- router projection (the reference of the router kernel) ------------------------------

def _bf16_bits(v):
    """bf16 bits of fp32 values that bf16 holds exactly (small integers, 0, 1)."""
    b = (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(synth.bf16_to_f32(b), np.asarray(v, np.float32))
    return b


def test_router_integer_case_equals_int64_matmul():
    # small integers are exact in bf16 (|v| <= 256) and fp32, and every partial
    # sum stays far below 2^53: the fp64 sum is exact and must equal numpy's
    # int64 matrix product plus the (integer) bias
    rng = np.random.default_rng(5)
    T, H, E = 7, 96, 5
    xi = rng.integers(-8, 9, size=(T, H))
    wi = rng.integers(-50, 51, size=(E, H))
    bi = rng.integers(-1000, 1001, size=E)
    got = oracle.router_logits(_bf16_bits(xi.astype(np.float32)), wi.astype(np.float32), bi.astype(np.float32))
    assert np.array_equal(got, (xi @ wi.T + bi).astype(np.float64))


def test_router_one_hot_rows_pick_weight_columns():
    # x[t] = e_{h_t}: S[t, e] = Wr[e, h_t] exactly (a transposed or shifted
    # operand fails this on a non-square shape); x = 0 gives the bias
    rng = np.random.default_rng(6)
    T, H, E = 5, 40, 3
    wr = rng.standard_normal((E, H)).astype(np.float32)
    hs = [0, 7, 39, 12, 7]
    x = np.zeros((T + 1, H), np.float32)
    for t, h in enumerate(hs):
        x[t, h] = 1.0
    b = rng.standard_normal(E).astype(np.float32)
    got = oracle.router_logits(_bf16_bits(x), wr, b)
    for t, h in enumerate(hs):
        assert np.array_equal(got[t], wr[:, h].astype(np.float64) + b.astype(np.float64))
    assert np.array_equal(got[T], b.astype(np.float64))
    assert np.array_equal(oracle.router_logits(_bf16_bits(x), wr)[T], np.zeros(E))


def test_router_matches_harness_logits(workload_data):
    # the harness rounds the same fp64 sum to fp32 once: they must agree to
    # within that rounding on a workload
    w = synth.WORKLOADS["tiny_T4"]
    d = workload_data("tiny_T4")
    wr = synth.router_weight(w.seed, w.E, w.H)
    got = oracle.router_logits(d["x"], wr)
    assert np.array_equal(got.astype(np.float32), d["logits"])


def test_route_matches_full_stable_sort_with_ties():
    rng = np.random.default_rng(3)
    for E, k in [(16, 2), (16, 16), (256, 6), (7, 3)]:
        l = rng.integers(-3, 4, (200, E)).astype(np.float32)  # many exact ties
        idx, gates = oracle.route(l, k)
        ref = np.argsort(-l, axis=1, kind="stable")[:, :k]      # ties -> lower id
        assert np.array_equal(idx, ref)
        assert np.allclose(gates.sum(1), 1.0, atol=1e-12)
        sel = np.take_along_axis(l, ref, 1).astype(np.float64)
        assert np.allclose(gates, scipy.special.softmax(sel, axis=1), rtol=1e-12)


def test_route_k_equals_E_is_full_softmax():
    rng = np.random.default_rng(4)
    l = rng.normal(0, 1.3, (50, 16)).astype(np.float32)
    idx, gates = oracle.route(l, 16)
    full = scipy.special.softmax(l.astype(np.float64), axis=1)
    assert np.allclose(gates, np.take_along_axis(full, idx, 1), rtol=1e-12)
    assert np.all(np.diff(np.take_along_axis(l, idx, 1), axis=1) <= 0)


def test_route_nan_ranks_last():
    l = np.float32([[np.nan, 1.0, 2.0, np.nan, -np.inf]])
    idx, _ = oracle.route(l, 5)
    assert list(idx[0]) == [2, 1, 4, 0, 3]


def test_route_invariants_on_workloads(workload_data):
    for name in ["tiny_T4", "decode_T8", "decode_T64"]:
        d = workload_data(name)
        k = synth.WORKLOADS[name].k
        idx, gates = oracle.route(d["logits"], k)
        assert np.all(gates > 0) and np.allclose(gates.sum(1), 1, atol=1e-12)
        assert all(len(set(r)) == k for r in idx)


# ---- sort ----------------------------------------------------------------------------

def test_sort_matches_numpy_stable_argsort():
    rng = np.random.default_rng(5)
    for T, k, E in [(4, 2, 16), (64, 6, 256), (1000, 6, 256), (1, 1, 1), (33, 3, 5)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, pos = oracle.sort(idx, E)
        flat = idx.ravel()
        assert np.array_equal(perm, np.argsort(flat, kind="stable"))
        assert np.array_equal(counts, np.bincount(flat, minlength=E))
        assert offsets[0] == 0 and offsets[-1] == T * k and np.all(np.diff(offsets) == counts)
        assert np.array_equal(pos[perm], np.arange(T * k))
        assert np.all(flat[perm] == np.repeat(np.arange(E), counts))


def test_sort_rejects_bad_expert_id():
    with pytest.raises(ValueError):
        oracle.sort(np.array([[0, 5]], np.int32), 5)
    with pytest.raises(ValueError):
        oracle.sort(np.array([[-1, 2]], np.int32), 5)


# ---- expert dot products ----------------------------------------------------------

def _random_rows(rng, n, K, smin, smax):
    q = rng.integers(-127, 128, (n, K)).astype(np.int8)
    c = rng.integers(0, 256, (n, K // 2)).astype(np.uint8)
    s = rng.integers(smin, smax + 1, (n, K // 32)).astype(np.uint8)
    return q, c, s


@pytest.mark.parametrize("smin,smax", [(120, 124), (100, 125), (0, 20), (230, 254)])
def test_dot_fp64_equals_int64_fixed_point(smin, smax):
    rng = np.random.default_rng(6)
    q, c, s = _random_rows(rng, 256, 4096, smin, smax)
    out, outf, ok = oracle.rows_dot(q, np.arange(256), c, s, np.arange(256))
    assert np.all(ok == 1)
    assert np.array_equal(out, outf)


def test_dot_fixed_point_reports_out_of_range_spans():
    # scale bytes of one row spanning 60 binades leave the exact fp64 domain;
    # the fixed-point reference says so instead of returning a rounded value
    rng = np.random.default_rng(6)
    q, c, s = _random_rows(rng, 64, 4096, 60, 120)
    _, _, ok = oracle.rows_dot(q, np.arange(64), c, s, np.arange(64))
    assert np.any(ok == 0)


def test_dot_matches_decoded_matmul():
    # decode with ml_dtypes, multiply with a float64 BLAS matmul: every term and
    # partial sum is exact, so the results must agree bit for bit.
    rng = np.random.default_rng(7)
    q, c, s = _random_rows(rng, 64, 2048, 118, 126)
    lo, hi = c & 15, c >> 4
    codes = np.stack([lo, hi], -1).reshape(64, 2048)
    w = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64) * np.repeat(
        s.view(ml_dtypes.float8_e8m0fnu).astype(np.float64), 32, axis=1)
    ref = np.einsum("rk,rk->r", q.astype(np.float64), w)
    got = oracle.rows_dot(q, np.arange(64), c, s, np.arange(64), fixed=False)
    assert np.array_equal(got, ref)


def test_dot_integer_special_case():
    # scale byte 127 and codes 2 (+1.0) / 10 (-1.0): the product is an integer
    # matrix product, checked against float64 matmul.
    rng = np.random.default_rng(8)
    K = 512
    q = rng.integers(-127, 128, (8, K)).astype(np.int8)
    sign = rng.integers(0, 2, (16, K))
    codes = np.where(sign == 1, 10, 2).astype(np.uint8)
    packed = (codes[:, 0::2] | (codes[:, 1::2] << 4)).astype(np.uint8)
    scales = np.full((16, K // 32), 127, np.uint8)
    ref = q.astype(np.float64) @ np.where(sign == 1, -1.0, 1.0).T
    qi = np.repeat(np.arange(8), 16)
    wi = np.tile(np.arange(16), 8)
    got = oracle.rows_dot(q, qi, packed, scales, wi, fixed=False).reshape(8, 16)
    assert np.array_equal(got, ref)


# ---- the whole layer ----------------------------------------------------------------

def _fwd(d, k, **kw):
    return oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                          d["w2_scales"], k, **kw)


def _make(T, H, E, k, I, seed, bias=0.0):
    return synth.make(synth.custom("t", T, H, E, k, I, seed, bias))


@pytest.mark.parametrize("T,H,E,k,I,seed", [(4, 256, 16, 2, 128, 0), (5, 128, 8, 3, 64, 11),
                                            (3, 64, 4, 4, 32, 12), (6, 96, 12, 1, 96, 13)])
def test_layer_equals_dense_mask_bruteforce(T, H, E, k, I, seed):
    d = synth.make(synth.WORKLOADS["tiny_T4"]) if seed == 0 else _make(T, H, E, k, I, seed)
    o = _fwd(d, k, want_Y=True)
    y64, y = oracle.forward_dense(d["x"], d["logits"], d["w1_codes"], d["w1_scales"],
                                  d["w2_codes"], d["w2_scales"], k)
    # fp64 sums of the same k terms in another order: equal to ~1 ulp of fp64
    ref64 = np.einsum("tj,tjn->tn", o["gates"], o["Y"].reshape(T, k, H).astype(np.float64))
    assert np.allclose(ref64, y64, rtol=1e-13, atol=1e-300)
    if k <= 2:
        assert np.array_equal(y, o["y"])
    else:
        assert np.mean(y == o["y"]) > 0.999


def test_layer_token_order_invariance():
    d = _make(12, 128, 8, 3, 64, 21)
    k = 3
    o = _fwd(d, k)
    p = np.random.default_rng(0).permutation(12)
    d2 = dict(d, x=np.ascontiguousarray(d["x"][p]), logits=np.ascontiguousarray(d["logits"][p]))
    o2 = _fwd(d2, k)
    assert np.array_equal(o2["y"], o["y"][p])
    assert np.array_equal(o2["xq"], o["xq"][p])
    assert np.array_equal(o2["hq"].reshape(12, k, -1), o["hq"].reshape(12, k, -1)[p])
    assert np.array_equal(o2["counts"], o["counts"])


def test_layer_single_expert_is_plain_quantised_mlp():
    # E = 1, k = 1: gate 1, no routing choice; the layer is a quantised SwiGLU
    # MLP, computed here with ml_dtypes decode, numpy fp32 quantisation and a
    # float64 matmul.
    T, H, I = 6, 128, 64
    d = _make(T, H, 1, 1, I, 31)
    o = _fwd(d, 1)
    assert np.all(o["gates"] == 1.0)

    def dec(codes, scales):
        n, kb = codes.shape
        c = np.stack([codes & 15, codes >> 4], -1).reshape(n, 2 * kb)
        return c.view(ml_dtypes.float4_e2m1fn).astype(np.float64) * np.repeat(
            scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64), 32, axis=1)

    def q8(v):
        a = np.abs(v).max(axis=1)
        s = (a / np.float32(127)).astype(np.float32)
        q = np.clip(np.rint(v / s[:, None]), -127, 127).astype(np.int8)
        return q, s

    W1, W2 = dec(d["w1_codes"][0], d["w1_scales"][0]), dec(d["w2_codes"][0], d["w2_scales"][0])
    x = synth.bf16_to_f32(d["x"])
    xq, sx = q8(x)
    assert np.array_equal(xq, o["xq"]) and np.array_equal(sx, o["sx"])
    G = (sx.astype(np.float64)[:, None] * (xq.astype(np.float64) @ W1.T)).astype(np.float32)
    g, u = G[:, :I].astype(np.float64), G[:, I:].astype(np.float64)
    h = (g * scipy.special.expit(g) * u).astype(np.float32)
    hq, sh = q8(h)
    assert np.abs(hq.astype(int) - o["hq"].astype(int)).max() <= 1
    assert np.allclose(sh, o["sh"], rtol=1e-6)
    Y = sh.astype(np.float64)[:, None] * (o["hq"].astype(np.float64) @ W2.T)
    yo = synth.bf16_to_f32(o["y"]).astype(np.float64)
    assert np.abs(yo - Y).max() <= 2 ** -8 * np.abs(Y).max()


def test_layer_invariants_decode_T8(workload_data):
    d = workload_data("decode_T8")
    o = _fwd(d, 6)
    assert o["counts"].sum() == 8 * 6
    assert np.allclose(o["gates"].sum(1), 1, atol=1e-12)
    assert np.all(np.abs(o["hq"]).max(1) == 127)
    assert np.all(np.abs(o["xq"]).max(1) == 127)


def test_forward_tokens_matches_forward(workload_data):
    d = workload_data("tiny_T4")
    o = _fwd(d, 2)
    ot = oracle.forward_tokens(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                               d["w2_scales"], 2, [2, 0])
    assert np.array_equal(ot["y"], o["y"][[2, 0]])
    assert np.array_equal(ot["hq"].reshape(2, 2, -1), o["hq"].reshape(4, 2, -1)[[2, 0]])
    assert np.array_equal(ot["sh"].reshape(2, 2), o["sh"].reshape(4, 2)[[2, 0]])


def _bf16_nearest_bruteforce(v: float) -> int:
    """Nearest bf16 to a double by exhaustive comparison of its two neighbours
    (ties to the even bit pattern); differences of nearby doubles are exact."""
    b = int(np.array([v], np.float32).view(np.uint32)[0] >> 16)  # truncation toward zero
    cands = [b, b + 1] if v >= 0 else [b, b + 1]
    vals = [float((np.array([c], np.uint32) << 16).view(np.float32)[0]) for c in cands]
    d = [abs(v - x) for x in vals]
    if d[0] != d[1]:
        return cands[0] if d[0] < d[1] else cands[1]
    return cands[0] if cands[0] % 2 == 0 else cands[1]


def test_bf16_rounding_of_double():
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.normal(0, 100, 3000), rng.normal(0, 1e-3, 1000),
                        1.0 + 2.0 ** -8 + rng.integers(-4, 5, 200) * 2.0 ** -40])
    for a in v:
        a = float(a)
        assert oracle.bf16_from_double(a) == _bf16_nearest_bruteforce(a), a
    # a double just above a bf16 tie: rounding through fp32 first would lose it
    assert oracle.bf16_from_double(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.bf16_from_double(1.0 + 2.0 ** -8) == 0x3F80   # exact tie -> even
    assert oracle.bf16_from_double(-(1.0 + 3 * 2.0 ** -8)) == 0xBF82  # tie -> even, negative
