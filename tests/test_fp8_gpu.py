"""The FP8 block-quantised dense projection (moe_fp8_*) against the oracle,
through the C ABI.

Bit-exact: the packed-layout round trip, the E4M3 codes and UE8M0 bytes of the
quantised activations.  Calls of at most 64 tokens split each tile's K range
over several CTAs (fp32 partial sums added in a fixed order): the same bound
holds.  Tolerance on the bf16 output (the layer's bar:
max|dy| <= 2e-2 max|y_oracle|, relative Frobenius error <= 5e-3), and per
element |y - y_exact| <= one bf16 ulp + 2^-12 * sum_k |terms| (fp32 tensor-core
accumulation of up to K exact products, then one bf16 rounding).
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

Y_MAX_REL = 2e-2
Y_FRO_REL = 5e-3


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _run(moe, d, N, tok=None):
    x = cu(d["x"]).view(torch.bfloat16)
    T, K = x.shape
    packed = moe.moe_fp8_pack_weights(cu(d["w_codes"]), cu(d["w_scales"]))
    dbg = dict(q=torch.empty((T, K), dtype=torch.uint8, device="cuda"),
               s=torch.empty((T, K // 128), dtype=torch.uint8, device="cuda"))
    ws = torch.empty(moe.lib.moe_fp8_workspace_bytes(T, N, K), dtype=torch.uint8, device="cuda")
    ybuf = torch.full((T + 2, N), 3.0, dtype=torch.bfloat16, device="cuda")
    y = ybuf[1:T + 1]
    moe.moe_fp8_linear(x, packed, N, ws=ws, y=y, debug=dbg)
    torch.cuda.synchronize()
    assert torch.all(ybuf[0] == 3.0) and torch.all(ybuf[T + 1] == 3.0), "output canary overwritten"
    assert moe.moe_check_device_flag(ws) == 0
    return y, dbg, packed, ws


def _check(y_gpu, q, s, d, tok=None):
    oq, os_ = oracle.fp8_quant_act(d["x"] if tok is None else d["x"][tok])
    qg, sg = q.cpu().numpy(), s.cpu().numpy()
    if tok is not None:
        qg, sg = qg[tok], sg[tok]
    assert np.array_equal(qg, oq), int((qg != oq).sum())
    assert np.array_equal(sg, os_)
    yo, y64, yabs = oracle.fp8_linear(oq, os_, d["w_codes"], d["w_scales"], want_f64=True)
    yg = y_gpu.float().cpu().numpy().astype(np.float64)
    if tok is not None:
        yg = yg[tok]
    yob = synth.bf16_to_f32(yo).astype(np.float64)
    m = np.abs(yob).max()
    assert np.abs(yg - yob).max() <= Y_MAX_REL * m
    assert np.linalg.norm(yg - yob) <= Y_FRO_REL * np.linalg.norm(yob)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y64), 1e-30))) - 7)
    assert np.all(np.abs(yg - y64) <= ulp + 2.0 ** -12 * yabs)
    return float(np.max(np.abs(yg - y64) / np.maximum(yabs, 1e-30)))


def test_fp8_pack_round_trip(moe):
    d = synth.fp8_weights(3, 256, 384)
    wq, ws = cu(d["w_codes"]), cu(d["w_scales"])
    packed = moe.moe_fp8_pack_weights(wq, ws)
    assert packed.numel() == moe.lib.moe_fp8_packed_bytes(256, 384)
    bq, bs = moe.moe_fp8_unpack_weights(packed, 256, 384)
    assert torch.equal(bq, wq) and torch.equal(bs, ws)
    ws[1, 2] = 0xFF
    with pytest.raises(moe.MoeError):
        moe.moe_fp8_pack_weights(wq, ws)


@pytest.mark.parametrize("T,N,K,seed", [
    (1, 128, 128, 1),        # one token, one block
    (130, 256, 384, 2),      # two token tiles, the second with 2 rows; 3 stages
    (300, 384, 512, 3),      # ragged: 44 rows in the last token tile
    (128, 128, 4096, 4),     # a full tile, 32 stages
    (37, 512, 256, 5),       # (calls of at most 64 tokens split the K range: here 2 ways)
    (8, 1024, 2048, 6),      # 8 weight tiles, K split 8 ways
    (64, 256, 384, 7),       # K split 3 ways over 3 stages: one stage each
    (65, 256, 512, 8),       # one token more: no split
])
def test_fp8_linear_shapes(moe, T, N, K, seed):
    d = dict(x=synth.x_bf16(seed, T, K))
    d.update(synth.fp8_weights(seed, N, K))
    x = d["x"].view(np.int16).copy()
    if T > 2:
        x[1, 128:256] = 0                                          # an all-zero block
        x[2, :128] = np.int16(0x0001)                              # bf16 subnormals
    d["x"] = x.view(np.uint16)
    y, dbg, _, _ = _run(moe, d, N)
    _check(y, dbg["q"], dbg["s"], d)


@pytest.mark.parametrize("name", ["dense_T8", "dense_T4604"])
def test_fp8_linear_workloads(moe, name):
    w = synth.DENSE_WORKLOADS[name]
    d = synth.make_dense(w)
    y, dbg, _, _ = _run(moe, d, w.N)
    if w.T <= 64:
        _check(y, dbg["q"], dbg["s"], d)
    else:
        # every token's codes whole; y on tokens from the first, a middle and the last token tile
        oq, os_ = oracle.fp8_quant_act(d["x"])
        assert np.array_equal(dbg["q"].cpu().numpy(), oq) and np.array_equal(dbg["s"].cpu().numpy(), os_)
        tok = np.array(sorted({0, 1, 127, 128, w.T // 2, w.T - 2, w.T - 1}), np.int64)
        _check(y, dbg["q"], dbg["s"], d, tok)


def test_fp8_layout_mismatch_flag(moe):
    d = dict(x=synth.x_bf16(7, 16, 256))
    d.update(synth.fp8_weights(7, 256, 256))
    packed = moe.moe_fp8_pack_weights(cu(d["w_codes"]), cu(d["w_scales"]))
    x = cu(d["x"]).view(torch.bfloat16)
    ws = torch.empty(moe.lib.moe_fp8_workspace_bytes(16, 128, 256), dtype=torch.uint8, device="cuda")
    y = torch.full((16, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_fp8_linear(x, packed, 128, ws=ws, y=y)           # packed for N = 256
    assert moe.moe_check_device_flag(ws) & moe.FLAG_LAYOUT
    assert torch.all(y == 5.0)
