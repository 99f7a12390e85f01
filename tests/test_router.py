"""The router projection kernel (moe_router_logits) against the oracle.

The bar is the fp32 summation bound, which holds for any summation order:
|logit - S| <= gamma_(H+1) * sum_h |x_h w_h| + u * |S| (+ the same slack), with
S the oracle's fp64 value, gamma_n = n u / (1 - n u) and u = 2^-24.  A wrong
index, a dropped or transposed operand exceeds it by orders of magnitude.
"""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _check(moe, x_bits, wr, bias):
    T, H = x_bits.shape
    got = moe.moe_router_logits(cu(x_bits).view(torch.bfloat16), cu(wr), None if bias is None else cu(bias))
    torch.cuda.synchronize()
    got = got.cpu().numpy().astype(np.float64)
    ref = oracle.router_logits(x_bits, wr, bias)
    xa = np.abs(synth.bf16_to_f32(x_bits).astype(np.float64))
    A = xa @ np.abs(wr.astype(np.float64)).T                 # sum_h |x_h w_h|
    n = H + 1
    gamma = n * U / (1 - n * U)
    bound = 1.01 * (gamma * A + U * (np.abs(ref) + gamma * A)) + 1e-30
    err = np.abs(got - ref)
    assert np.all(err <= bound), float((err / bound).max())
    return float((err / np.maximum(np.abs(ref), 1e-30)).max())


@pytest.mark.parametrize("name", ["tiny_T4", "decode_T8", "decode_T64", "prefill_T4604"])
def test_router_matches_oracle_on_workloads(moe, workload_data, name):
    w = synth.WORKLOADS[name]
    d = workload_data(name)
    wr = synth.router_weight(w.seed, w.E, w.H)
    _check(moe, d["x"], wr, None)


def test_router_with_bias_skewed_prefill_rows(moe):
    # the skewed workload's bias b_e = 3 ln(1/(e+1)), on a slice of its tokens
    w = synth.WORKLOADS["prefill_skew_T16384"]
    x = synth.x_bf16(w.seed, 300, w.H)
    wr = synth.router_weight(w.seed, w.E, w.H)
    bias = synth.router_bias(w.E, w.bias_coef).astype(np.float32)
    _check(moe, x, wr, bias)


@pytest.mark.parametrize("T,H,E", [(1, 32, 1), (65, 160, 65), (3, 128, 1024), (130, 96, 7),
                                   (16, 4096, 256), (17, 4096, 256), (5, 288, 9)])
def test_router_ragged_shapes(moe, T, H, E):
    # tiles of 64 tokens x 64 experts with ragged edges on both sides; up to
    # 16 tokens the warp-per-expert kernel (E not a multiple of its 8 warps)
    rng = np.random.default_rng(T * 7 + E)
    x = synth.x_bf16(11 + T, T, H)
    wr = (0.02 * rng.standard_normal((E, H))).astype(np.float32)
    bias = rng.standard_normal(E).astype(np.float32)
    _check(moe, x, wr, bias)


def test_router_zero_tokens_and_bad_args(moe):
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    wr = torch.zeros((4, 128), dtype=torch.float32, device="cuda")
    assert moe.moe_router_logits(x, wr).shape == (0, 4)
    with pytest.raises(moe.MoeError):
        moe.moe_router_logits(torch.empty((2, 100), dtype=torch.bfloat16, device="cuda"),
                              torch.zeros((4, 100), dtype=torch.float32, device="cuda"))


@pytest.mark.parametrize("T,H,E,k,I,seed", [(8, 4096, 256, 6, 2048, 1), (300, 512, 8, 2, 256, 81)])
def test_layer_with_router_equals_the_two_calls(moe, T, H, E, k, I, seed):
    # moe_layer_forward_with_router = moe_router_logits then moe_layer_forward,
    # bit for bit (decode-size fused front, and a call with tensor-core experts)
    w = synth.custom("lr", T, H, E, k, I, seed, 0.8 if T > 8 else 0.0)
    d = synth.make(w)
    wr = cu(synth.router_weight(seed, E, H))
    bias = cu(synth.router_bias(E, w.bias_coef).astype(np.float32)) if w.bias_coef else None
    packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]), cu(d["w2_scales"]))
    x = cu(d["x"]).view(torch.bfloat16)
    y1 = moe.moe_layer_forward_with_router(x, wr, bias, packed, H, I, E, k)
    logits = moe.moe_router_logits(x, wr, bias)
    ws = torch.empty(moe.moe_layer_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    y2 = moe.moe_layer_forward(logits, x, packed, H, I, E, k, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_check_device_flag(ws) == 0
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
