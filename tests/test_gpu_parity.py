"""CUDA path vs the CPU oracle, through the C ABI (libmoe.so).

Bit-exact: routing indices, sort permutation/positions/offsets, INT8 codes and
scales of x and h, packed-layout round trip.  Tolerance on the bf16 output
(max|dy| <= 2e-2 * max|y_oracle|, relative Frobenius error <= 5e-3) and on the
fp32 gates (1e-6 relative to the oracle's fp64 gates).
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
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


_orc_cache = {}


def oracle_full(name, d):
    if name not in _orc_cache:
        w = synth.WORKLOADS[name]
        _orc_cache[name] = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"],
                                          d["w2_codes"], d["w2_scales"], w.k)
    return _orc_cache[name]


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def effective_tc_threshold(moe, T):
    """The tensor-core row threshold a call of T tokens uses (MOE_OPT_TC_MIN_ROWS;
    0 = automatic: every expert streams below 32 tokens, else 2)."""
    v = moe.moe_get_option(moe.MOE_OPT_TC_MIN_ROWS)
    if v > 0:
        return v
    return 2 ** 31 - 1 if T < 32 else 2


def y_check(y_gpu_bf16, y_orc_bits):
    yg = y_gpu_bf16.float().cpu().numpy().astype(np.float64)
    yo = synth.bf16_to_f32(y_orc_bits).astype(np.float64)
    m = np.abs(yo).max()
    assert np.abs(yg - yo).max() <= Y_MAX_REL * m, (np.abs(yg - yo).max(), m)
    fro = np.linalg.norm(yg - yo) / max(np.linalg.norm(yo), 1e-300)
    assert fro <= Y_FRO_REL, fro
    return np.abs(yg - yo).max() / m, fro


def run_layer(moe, d, w, debug=True):
    H, I, E, k = w.H, w.I, w.E, w.k
    T = d["x"].shape[0]
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                  cu(d["w2_scales"]))
    logits = cu(d["logits"])
    idx, gates = moe.moe_route(logits, k)
    perm, pos, offsets = moe.moe_sort(idx, E)
    x = cu(d["x"]).view(torch.bfloat16)
    dbg = None
    if debug:
        dbg = dict(xq=torch.empty((T, H), dtype=torch.int8, device="cuda"),
                   sx=torch.empty(T, dtype=torch.float32, device="cuda"),
                   hq=torch.empty((T * k, I), dtype=torch.int8, device="cuda"),
                   sh=torch.empty(T * k, dtype=torch.float32, device="cuda"))
    ws = torch.empty(moe.moe_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    # canary rows around the output
    ybuf = torch.full((T + 2, H), 7.0, dtype=torch.bfloat16, device="cuda")
    y = ybuf[1:T + 1]
    moe.moe_forward(x, idx, gates, perm, pos, offsets, packed, H, I, E, ws=ws, y=y, debug=dbg)
    torch.cuda.synchronize()
    assert torch.all(ybuf[0] == 7.0) and torch.all(ybuf[T + 1] == 7.0), "output canary overwritten"
    assert moe.moe_check_device_flag(ws) == 0
    return dict(idx=idx, gates=gates, perm=perm, pos=pos, offsets=offsets, y=y, dbg=dbg,
                packed=packed)


# ---- packing ------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny_T4", "decode_T8"])
def test_pack_unpack_round_trip(moe, workload_data, name):
    d, w = workload_data(name), synth.WORKLOADS[name]
    canon = [cu(d[n]) for n in ("w1_codes", "w1_scales", "w2_codes", "w2_scales")]
    packed = moe.moe_pack_weights(*canon)
    assert packed.numel() == moe.moe_packed_bytes(w.H, w.I, w.E)
    back = moe.moe_unpack_weights(packed, w.H, w.I, w.E)
    for a, b in zip(canon, back):
        assert torch.equal(a, b)


def test_pack_covers_all_byte_values(moe):
    # every code byte 0..255 and every legal scale byte 0..254 survives the round trip
    E, H, I = 2, 256, 128
    rng = np.random.default_rng(0)
    w1c = np.resize(np.arange(256, dtype=np.uint8), (E, 2 * I, H // 2))
    w1s = np.resize(np.arange(255, dtype=np.uint8), (E, 2 * I, H // 32))
    w2c = rng.integers(0, 256, (E, H, I // 2), dtype=np.uint8)
    w2s = np.resize(np.arange(255, dtype=np.uint8)[::-1].copy(), (E, H, I // 32))
    canon = [cu(a) for a in (w1c, w1s, w2c, w2s)]
    back = moe.moe_unpack_weights(moe.moe_pack_weights(*canon), H, I, E)
    for a, b in zip(canon, back):
        assert torch.equal(a, b)


def test_pack_rejects_nan_scale(moe):
    E, H, I = 1, 128, 128
    w1c = torch.zeros((E, 2 * I, H // 2), dtype=torch.uint8, device="cuda")
    w1s = torch.full((E, 2 * I, H // 32), 127, dtype=torch.uint8, device="cuda")
    w2c = torch.zeros((E, H, I // 2), dtype=torch.uint8, device="cuda")
    w2s = torch.full((E, H, I // 32), 127, dtype=torch.uint8, device="cuda")
    w2s[0, 5, 1] = 0xFF
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_pack_weights(w1c, w1s, w2c, w2s)
    assert ei.value.status == -1


def test_mispermuted_w2_layout_is_caught(moe, workload_data):
    # The layout bug of the paper: W2 rows permuted in the device layout.  Both
    # the unpack round trip and the comparison with the oracle must catch it.
    name = "tiny_T4"
    d, w = workload_data(name), synth.WORKLOADS[name]
    r = run_layer(moe, d, w, debug=False)
    packed = r["packed"]
    # swap the code pieces of rows 0 and 1 of every 128-row block of one used
    # expert's W2 (packed chunk of 8704 bytes: 512 scale bytes, then for each
    # of 4 blocks the 128 rows' 16-byte pieces)
    e = int(r["idx"][0, 0])
    w2_off = 256 + w.E * (2 * w.I * w.H * 17 // 32) + e * (w.H * w.I * 17 // 32)
    KG = w.I // 128
    for rb in range(w.H // 128):
        for g in range(KG):
            for j in range(4):
                o = w2_off + (rb * KG + g) * 8704 + 512 + j * 2048
                a = packed[o:o + 16].clone()
                packed[o:o + 16] = packed[o + 16:o + 32]
                packed[o + 16:o + 32] = a
    back = moe.moe_unpack_weights(packed, w.H, w.I, w.E)
    assert not torch.equal(back[2], cu(d["w2_codes"]))
    x = cu(d["x"]).view(torch.bfloat16)
    y = moe.moe_forward(x, r["idx"], r["gates"], r["perm"], r["pos"], r["offsets"], packed,
                        w.H, w.I, w.E)
    o = oracle_full(name, d)
    with pytest.raises(AssertionError):
        y_check(y, o["y"])


# ---- routing -------------------------------------------------------------------------

@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_route_parity(moe, name):
    w = synth.WORKLOADS[name]
    d = synth.activations(w)
    idx, gates = moe.moe_route(cu(d["logits"]), w.k)
    oi, og = oracle.route(d["logits"], w.k)
    assert np.array_equal(idx.cpu().numpy(), oi)
    g = gates.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(g - og) <= GATE_REL * og + 1e-12)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (37, 16, 16), (100, 256, 6), (5, 1024, 16),
                                   (64, 300, 7), (0, 8, 2)])
def test_route_edge_cases(moe, T, E, k):
    rng = np.random.default_rng(T * 1000 + E)
    l = rng.integers(-2, 3, (T, E)).astype(np.float32)  # heavy ties
    if T > 3:
        l[1, :] = 0.0
        l[2, ::3] = np.nan
        l[3, 0] = -np.inf
    idx, gates = moe.moe_route(cu(l), k) if T else moe.moe_route(torch.empty((0, E), device="cuda"), k)
    if T == 0:
        return
    oi, og = oracle.route(l, k)
    assert np.array_equal(idx.cpu().numpy(), oi)
    g = gates.cpu().numpy().astype(np.float64)
    ok = np.isfinite(og)
    assert np.all(np.abs(g[ok] - og[ok]) <= GATE_REL * og[ok] + 1e-12)


# ---- sort ---------------------------------------------------------------------------------

@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_sort_parity(moe, name):
    w = synth.WORKLOADS[name]
    d = synth.activations(w)
    oi, _ = oracle.route(d["logits"], w.k)
    perm, pos, offsets = moe.moe_sort(cu(oi), w.E)
    counts, ooff, operm, opos = oracle.sort(oi, w.E)
    assert np.array_equal(offsets.cpu().numpy(), ooff)
    assert np.array_equal(perm.cpu().numpy(), operm)
    assert np.array_equal(pos.cpu().numpy(), opos)


@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (512, 2, 3), (171, 6, 256), (1024, 1, 16),
                                   (1025, 1, 16), (683, 3, 1024), (20000, 6, 256), (0, 6, 256)])
def test_sort_sizes(moe, T, k, E):
    rng = np.random.default_rng(T + k + E)
    idx = np.zeros((T, k), np.int32)
    for t in range(T):
        idx[t] = rng.permutation(E)[:k]
    if T >= 100:  # skew: half the pairs on one expert
        idx[: T // 2, 0] = E - 1 if k == 1 else idx[: T // 2, 0]
    perm, pos, offsets = moe.moe_sort(cu(idx), E)
    counts, ooff, operm, opos = oracle.sort(idx, E)
    assert np.array_equal(offsets.cpu().numpy(), ooff)
    assert np.array_equal(perm.cpu().numpy(), operm)
    assert np.array_equal(pos.cpu().numpy(), opos)


def test_sort_flags_bad_expert(moe):
    idx = torch.tensor([[0, 1], [2, 9]], dtype=torch.int32, device="cuda")
    ws = torch.empty(moe.moe_sort_workspace_bytes(2, 2, 4), dtype=torch.uint8, device="cuda")
    moe.moe_sort(idx, 4, ws=ws)
    assert moe.moe_check_device_flag(ws) & moe.FLAG_BAD_EXPERT


# ---- quantisation stage ----------------------------------------------------------------

def test_quant_rows_stage(moe):
    rng = np.random.default_rng(3)
    v = rng.normal(0, 5, (300, 2048)).astype(np.float32)
    v[0] = 0.0
    v[1, :4] = [127.0, 0.5, 1.5, -2.5]
    v[1, 4:] = 0.0
    v[2] = np.float32(1e-30) * rng.normal(size=2048).astype(np.float32)
    q, s = moe.moe_quant_rows_f32(cu(v))
    oq, os_ = oracle.quant_rows(v)
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(s.cpu().numpy(), os_)


# ---- the whole layer --------------------------------------------------------------------

def _check_layer(moe, d, w, o):
    r = run_layer(moe, d, w)
    T, k = d["x"].shape[0], w.k
    assert np.array_equal(r["idx"].cpu().numpy(), o["idx"])
    assert np.array_equal(r["perm"].cpu().numpy(), o["perm"])
    assert np.array_equal(r["offsets"].cpu().numpy(), o["offsets"])
    assert np.array_equal(r["dbg"]["xq"].cpu().numpy(), o["xq"])
    assert np.array_equal(r["dbg"]["sx"].cpu().numpy(), o["sx"])
    perm = o["perm"]
    hq = r["dbg"]["hq"].cpu().numpy()
    sh = r["dbg"]["sh"].cpu().numpy()
    assert np.array_equal(hq, o["hq"][perm]), int((hq != o["hq"][perm]).sum())
    assert np.array_equal(sh, o["sh"][perm])
    return y_check(r["y"], o["y"])


@pytest.mark.parametrize("name", ["tiny_T4", "decode_T8", "decode_T64"])
def test_forward_parity_full(moe, workload_data, name):
    d, w = workload_data(name), synth.WORKLOADS[name]
    _check_layer(moe, d, w, oracle_full(name, d))


@pytest.mark.parametrize("T,H,E,k,I,seed", [
    (1, 128, 4, 1, 128, 41),      # single token, single expert
    (13, 384, 9, 3, 256, 42),     # ragged: 39 pairs, tiles of 32 rows over 384 inputs
    (9, 256, 16, 16, 128, 43),    # k = E: every expert gets every token
    (40, 256, 2, 2, 384, 44),     # 40 rows per expert: several token groups
    (3, 128, 1, 1, 128, 45),      # E = 1
])
def test_forward_parity_shapes(moe, T, H, E, k, I, seed):
    w = synth.custom("s", T, H, E, k, I, seed)
    d = synth.make(w)
    o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                       d["w2_scales"], k)
    _check_layer(moe, d, w, o)


def test_forward_zero_tokens(moe):
    H, I, E, k = 128, 128, 4, 2
    w = synth.custom("z", 1, H, E, k, I, 5)
    d = synth.make(w)
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                  cu(d["w2_scales"]))
    x = torch.empty((0, H), dtype=torch.bfloat16, device="cuda")
    idx = torch.empty((0, k), dtype=torch.int32, device="cuda")
    gates = torch.empty((0, k), dtype=torch.float32, device="cuda")
    perm, pos, offsets = moe.moe_sort(idx, E)
    assert torch.all(offsets == 0)
    y = moe.moe_forward(x, idx, gates, perm, pos, offsets, packed, H, I, E)
    assert y.shape == (0, H)


def test_forward_layout_mismatch_flag(moe):
    # weights packed for E=4 used as E=2: the header check raises FLAG_LAYOUT and
    # the GEMMs do not read the packed buffer
    w = synth.custom("m", 2, 128, 4, 2, 128, 6)
    d = synth.make(w)
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                  cu(d["w2_scales"]))
    idx, gates = moe.moe_route(cu(d["logits"][:, :2].copy()), 2)
    perm, pos, offsets = moe.moe_sort(idx, 2)
    ws = torch.empty(moe.moe_workspace_bytes(2, 128, 128, 2, 2), dtype=torch.uint8, device="cuda")
    moe.moe_forward(cu(d["x"]).view(torch.bfloat16), idx, gates, perm, pos, offsets, packed,
                    128, 128, 2, ws=ws)
    assert moe.moe_check_device_flag(ws) & moe.FLAG_LAYOUT


def test_forward_rejects_bad_args(moe):
    with pytest.raises(moe.MoeError):
        moe.moe_workspace_bytes(4, 100, 128, 4, 2)
    with pytest.raises(moe.MoeError):
        moe.moe_workspace_bytes(4, 128, 128, 4, 5)


def chosen_tokens(offsets, perm, k, T, n_total=256, seed=7):
    """Tokens for a sampled comparison, chosen to cover the layer's structure:
    the token of the first sorted row of every touched expert (so every
    expert, streaming or tensor-core, is hit), the token of the last row of 32
    of them (ragged tails), the tokens of the first, a middle and the last
    128-row token tile of the largest expert, the first and last token, then
    seeded random tokens up to n_total (the oracle evaluates each token
    separately)."""
    counts = np.diff(offsets)
    tok = {0, T - 1}
    touched = np.nonzero(counts)[0]
    for e in touched:
        tok.add(int(perm[offsets[e]]) // k)
    for e in touched[:: max(1, len(touched) // 32)]:
        tok.add(int(perm[offsets[e + 1] - 1]) // k)
    big = int(np.argmax(counts))
    nblk = (int(counts[big]) + 127) // 128
    for b in sorted({0, nblk // 2, nblk - 1}):
        r0 = offsets[big] + 128 * b
        r1 = min(offsets[big + 1], r0 + 128)
        tok.update(int(perm[r]) // k for r in (r0, (r0 + r1) // 2, r1 - 1))
    rng = np.random.default_rng(seed)
    while len(tok) < n_total:
        tok.add(int(rng.integers(0, T)))
    return np.array(sorted(tok), np.int32)


@pytest.mark.parametrize("name", ["prefill_T4604", "prefill_skew_T16384", "prefill_skew1.25_T16384"])
def test_forward_parity_sampled_full_size(moe, workload_data, name):
    """Full-size prefill workloads in the default configuration (experts at or
    above the automatic threshold on the tensor-core GEMM, the others on the
    streaming GEMM): every routing/sort value is compared whole; the layer's outputs on
    chosen tokens (every touched expert, the largest expert's first, middle and
    last token tile) are compared with the oracle's per-token computation
    (INT8 codes bit-exact, y within tolerance)."""
    d, w = workload_data(name), synth.WORKLOADS[name]
    r = run_layer(moe, d, w)
    oi, og = oracle.route(d["logits"], w.k)
    assert np.array_equal(r["idx"].cpu().numpy(), oi)
    counts, ooff, operm, opos = oracle.sort(oi, w.E)
    assert np.array_equal(r["perm"].cpu().numpy(), operm)
    assert np.array_equal(r["offsets"].cpu().numpy(), ooff)
    tok = chosen_tokens(ooff, operm, w.k, w.T)
    ot = oracle.forward_tokens(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                               d["w2_scales"], w.k, tok)
    assert np.array_equal(r["dbg"]["xq"].cpu().numpy()[tok], ot["xq"])
    assert np.array_equal(r["dbg"]["sx"].cpu().numpy()[tok], ot["sx"])
    pairs = (tok[:, None] * w.k + np.arange(w.k)[None, :]).ravel()
    rows = opos[pairs]
    # both kernels are covered wherever the workload has both kinds of expert
    thr = effective_tc_threshold(moe, w.T)
    tc_rows = counts[oi.ravel()[pairs]] >= thr
    if ((counts > 0) & (counts < thr)).any():
        assert (~tc_rows).any()
    assert tc_rows.any()
    assert np.array_equal(r["dbg"]["hq"].cpu().numpy()[rows], ot["hq"])
    assert np.array_equal(r["dbg"]["sh"].cpu().numpy()[rows], ot["sh"])
    y_check(r["y"][torch.from_numpy(tok).long().cuda()], ot["y"])


# ---- the layer's exp and SwiGLU, bit for bit ---------------------------------------

def test_exp_bit_identical_to_oracle(moe):
    # 2^24 bit patterns spread over the whole fp32 range, plus dense sweeps of
    # the interesting interval and the special values
    bits = (np.arange(1 << 24, dtype=np.uint64) * 256 + 77).astype(np.uint32)
    x = np.concatenate([bits.view(np.float32), np.linspace(-110, 95, 1 << 22, dtype=np.float32),
                        np.float32([0.0, -0.0, np.inf, -np.inf, np.nan, 88.8, -104.0, 88.72283])])
    y = moe.moe_exp_f32(cu(x)).cpu().numpy()
    ref = oracle.exp_f32(x)
    same = (y.view(np.uint32) == ref.view(np.uint32)) | (np.isnan(y) & np.isnan(ref))
    assert same.all(), int((~same).sum())


def test_swiglu_bit_identical_to_oracle(moe):
    rng = np.random.default_rng(11)
    g = np.concatenate([rng.normal(0, 10, 200000), rng.uniform(-120, 120, 50000)]).astype(np.float32)
    u = rng.normal(0, 10, g.size).astype(np.float32)
    h = moe.moe_swiglu_f32(cu(g), cu(u)).cpu().numpy()
    ref = np.array([oracle.swiglu(float(a), float(b)) for a, b in zip(g[:20000], u[:20000])],
                   np.float32)
    assert np.array_equal(h[:20000].view(np.uint32), ref.view(np.uint32))


# ---- the tensor-core grouped GEMM, forced on for every expert ------------------

@pytest.fixture
def tc_everywhere(moe):
    old = moe.moe_get_option(moe.MOE_OPT_TC_MIN_ROWS)
    moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, 1)
    yield
    moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, old)


@pytest.mark.parametrize("T,H,E,k,I,seed", [
    (40, 256, 2, 1, 128, 51),      # one n-block per expert, ragged (19/21 rows)
    (300, 512, 4, 2, 256, 52),     # several n-blocks per expert, ragged tails
    (13, 384, 9, 3, 256, 42),      # tiny experts: n_mma = 16
    (9, 256, 16, 16, 128, 43),     # k = E
    (257, 128, 1, 1, 128, 53),     # E = 1, 257 rows: three n-blocks, last holds one row
    # calls of more than 64 tokens: W1 token-major (256-row weight blocks), W2
    # weight-major; both token-major in tests/test_tc_forms.py
    (300, 384, 4, 2, 256, 54),     # H = 384: W2 with three 128-row weight blocks
    (130, 640, 3, 3, 384, 56),     # W1 N = 768 (three 256-row blocks), W2 N = 640
    (65, 256, 64, 2, 128, 57),     # one token row more than the decode configuration takes
])
def test_tc_forward_parity_shapes(moe, tc_everywhere, T, H, E, k, I, seed):
    w = synth.custom("tc", T, H, E, k, I, seed)
    d = synth.make(w)
    o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                       d["w2_scales"], k)
    _check_layer(moe, d, w, o)


def test_tc_forward_parity_decode_T64(moe, workload_data, tc_everywhere):
    # decode-shaped experts (1-7 rows) through the tensor-core path
    name = "decode_T64"
    d, w = workload_data(name), synth.WORKLOADS[name]
    _check_layer(moe, d, w, oracle_full(name, d))


def test_tc_option_validation(moe):
    with pytest.raises(moe.MoeError):
        moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, -1)
    with pytest.raises(moe.MoeError):
        moe.moe_set_option(99, 1)
    assert moe.moe_get_option(moe.MOE_OPT_TC_MIN_ROWS) >= 0


def test_forward_with_garbage_tables_raises_bounds_flag(moe):
    # perm/pos/topk_idx that did not come from moe_sort: every index is checked
    # inside the kernels, so the call completes and reports FLAG_BOUNDS
    w = synth.custom("g", 6, 128, 4, 2, 128, 61)
    d = synth.make(w)
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                  cu(d["w2_scales"]))
    idx, gates = moe.moe_route(cu(d["logits"]), 2)
    perm, pos, offsets = moe.moe_sort(idx, 4)
    bad = torch.full_like(perm, 1 << 20)
    ws = torch.empty(moe.moe_workspace_bytes(6, 128, 128, 4, 2), dtype=torch.uint8, device="cuda")
    moe.moe_forward(cu(d["x"]).view(torch.bfloat16), idx, gates, bad, bad, offsets, packed, 128, 128, 4,
                    ws=ws)
    assert moe.moe_check_device_flag(ws) & moe.FLAG_BOUNDS
    bad_off = offsets.clone()
    bad_off[2] = 10 ** 6
    moe.moe_forward(cu(d["x"]).view(torch.bfloat16), idx, gates, perm, pos, bad_off, packed, 128, 128, 4,
                    ws=ws)
    assert moe.moe_check_device_flag(ws) & moe.FLAG_BOUNDS
