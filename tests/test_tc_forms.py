"""The tensor-core grouped GEMM's alternative forms against the default forms
(for calls of more than 64 tokens W1 token-major and W2 weight-major; the
weight-major decode configuration below) and the oracle:

* both GEMMs weight-major (MOE_OPT_TC_FORM = 1: 128 weight rows as the MMA's
  M, 128 token rows as its N, one CTA per SM) or both token-major
  (MOE_OPT_TC_FORM = 2: 128 token rows as M, two 128-row weight chunks as N);
* SM pairs (MOE_OPT_TC_PAIR = 1: clusters of two CTAs, tcgen05 cta_group::2,
  M = 256), where the weight rows of a matrix are a multiple of 256 (W1
  always, W2 when H is); other shapes fall back to one CTA per SM, which a
  case here covers too;
* the weight operand staged in tensor memory (MOE_OPT_TC_A_TMEM = 1: one
  tcgen05.cp per stage, the digit-plane MMAs read A from TMEM).

All forms compute the same exact sums, so y, hq and sh must be bit-identical
between them; against the oracle the layer's usual bar applies (bit-exact
INT8 codes and scales, y within tolerance).
"""
import numpy as np
import pytest
import torch

import oracle
import synth

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


def _run(moe, d, w, pair, a_tmem=False, form=0):
    T, H, I, E, k = w.T, w.H, w.I, w.E, w.k
    keys = (moe.MOE_OPT_TC_MIN_ROWS, moe.MOE_OPT_TC_PAIR, moe.MOE_OPT_TC_A_TMEM, moe.MOE_OPT_TC_FORM)
    old = tuple(moe.moe_get_option(k_) for k_ in keys)
    moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, 1)
    moe.moe_set_option(moe.MOE_OPT_TC_PAIR, 1 if pair else 0)
    moe.moe_set_option(moe.MOE_OPT_TC_A_TMEM, 1 if a_tmem else 0)
    moe.moe_set_option(moe.MOE_OPT_TC_FORM, form)
    try:
        packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                      cu(d["w2_scales"]))
        idx, gates = moe.moe_route(cu(d["logits"]), k)
        perm, pos, offsets = moe.moe_sort(idx, E)
        dbg = dict(xq=torch.empty((T, H), dtype=torch.int8, device="cuda"),
                   sx=torch.empty(T, dtype=torch.float32, device="cuda"),
                   hq=torch.empty((T * k, I), dtype=torch.int8, device="cuda"),
                   sh=torch.empty(T * k, dtype=torch.float32, device="cuda"))
        ws = torch.empty(moe.moe_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device="cuda")
        y = moe.moe_forward(cu(d["x"]).view(torch.bfloat16), idx, gates, perm, pos, offsets, packed, H, I, E,
                            ws=ws, debug=dbg)
        torch.cuda.synchronize()
        assert moe.moe_check_device_flag(ws) == 0
        return y, dbg
    finally:
        for k_, v in zip(keys, old):
            moe.moe_set_option(k_, v)


@pytest.mark.parametrize("T,H,E,k,I,seed", [
    (40, 256, 2, 1, 128, 71),      # W1 and W2 in pairs; one token tile per expert, ragged
    (300, 512, 4, 2, 256, 72),     # several token tiles per expert, ragged tails
    (9, 256, 16, 16, 128, 73),     # k = E: 16 experts, tiny token tiles (n_mma = 16)
    (13, 384, 9, 3, 256, 74),      # H = 384: W2 falls back to one CTA per SM, W1 in pairs
    (257, 256, 1, 1, 128, 75),     # E = 1, three token tiles, the last holds one row
    (300, 384, 4, 2, 256, 76),     # token-major W2 with a ragged 128-row weight block
])
@pytest.mark.parametrize("form", ["pair", "a_tmem", "weight_major", "token_major"])
def test_form_matches_single_and_oracle(moe, form, T, H, E, k, I, seed):
    w = synth.custom("pair", T, H, E, k, I, seed)
    d = synth.make(w)
    y1, d1 = _run(moe, d, w, pair=False)
    y2, d2 = _run(moe, d, w, pair=form == "pair", a_tmem=form == "a_tmem",
                  form={"weight_major": 1, "token_major": 2}.get(form, 0))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    assert torch.equal(d1["hq"], d2["hq"])
    assert torch.equal(d1["sh"].view(torch.int32), d2["sh"].view(torch.int32))
    o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"], d["w2_scales"], k)
    perm = o["perm"]
    assert np.array_equal(d2["hq"].cpu().numpy(), o["hq"][perm])
    assert np.array_equal(d2["sh"].cpu().numpy(), o["sh"][perm])
    yg = y2.float().cpu().numpy().astype(np.float64)
    yo = synth.bf16_to_f32(o["y"]).astype(np.float64)
    m = np.abs(yo).max()
    assert np.abs(yg - yo).max() <= Y_MAX_REL * m
    assert np.linalg.norm(yg - yo) / max(np.linalg.norm(yo), 1e-300) <= Y_FRO_REL


def test_form_option_validation(moe):
    for opt in (moe.MOE_OPT_TC_PAIR, moe.MOE_OPT_TC_A_TMEM):
        with pytest.raises(moe.MoeError):
            moe.moe_set_option(opt, 2)
        assert moe.moe_get_option(opt) in (0, 1)
    for bad in (-1, 3):
        with pytest.raises(moe.MoeError):
            moe.moe_set_option(moe.MOE_OPT_TC_FORM, bad)
    assert moe.moe_get_option(moe.MOE_OPT_TC_FORM) in (0, 1, 2)
