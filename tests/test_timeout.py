"""The tensor-core GEMM's bounded waits, made to run out on purpose.

Every mbarrier wait inside the tensor-core grouped GEMM gives up after
MOE_OPT_WAIT_LIMIT_US and raises MOE_FLAG_TIMEOUT in the call's device error
word; the kernel then waits (bounded) for its own copies and MMAs, frees its
tensor memory and returns, so the process and the GPU stay usable.  The test
arms MOE_OPT_TEST_TIMEOUT, which makes the next tensor-core W1 launch withhold
its first CTA's first pipeline stage (no copy and no arrival: a barrier that
nothing completes), with a short limit so the wait ends in milliseconds.  It
expects the flag, then runs the same call normally in the same process and
checks it bit-exact against the oracle.  Nothing faults, traps or hangs.
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from tests.test_gpu_parity import _check_layer, cu  # noqa: E402


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


# the W1 kernel whose stage is withheld: weight-major decode configuration
# (40 tokens, form 1), weight-major prefill configuration (100 tokens, form 1),
# token-major (form 0)
@pytest.mark.parametrize("T,form", [(40, 1), (100, 1), (100, 0)])
def test_withheld_stage_times_out_then_next_call_is_exact(moe, T, form):
    keys = [moe.MOE_OPT_TC_MIN_ROWS, moe.MOE_OPT_TC_PAIR, moe.MOE_OPT_WAIT_LIMIT_US,
            moe.MOE_OPT_TEST_TIMEOUT, moe.MOE_OPT_TC_FORM]
    old = {k_: moe.moe_get_option(k_) for k_ in keys}
    w = synth.custom("to", T, 256, 2, 1, 128, 51)
    d = synth.make(w)
    try:
        moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, 1)
        moe.moe_set_option(moe.MOE_OPT_TC_PAIR, 0)
        moe.moe_set_option(moe.MOE_OPT_TC_FORM, form)
        moe.moe_set_option(moe.MOE_OPT_WAIT_LIMIT_US, 20000)   # 20 ms
        packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                      cu(d["w2_scales"]))
        idx, gates = moe.moe_route(cu(d["logits"]), w.k)
        perm, pos, offsets = moe.moe_sort(idx, w.E)
        ws = torch.empty(moe.moe_workspace_bytes(w.T, w.H, w.I, w.E, w.k), dtype=torch.uint8, device="cuda")
        moe.moe_set_option(moe.MOE_OPT_TEST_TIMEOUT, 1)
        moe.moe_forward(cu(d["x"]).view(torch.bfloat16), idx, gates, perm, pos, offsets, packed,
                        w.H, w.I, w.E, ws=ws)
        torch.cuda.synchronize()
        flag = moe.moe_check_device_flag(ws)
        assert flag & moe.FLAG_TIMEOUT, hex(flag)
        assert moe.moe_get_option(moe.MOE_OPT_TEST_TIMEOUT) == 0   # consumed by that call
        # the same process and GPU: a normal call is exact again
        moe.moe_set_option(moe.MOE_OPT_WAIT_LIMIT_US, old[moe.MOE_OPT_WAIT_LIMIT_US])
        o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                           d["w2_scales"], w.k)
        _check_layer(moe, d, w, o)
    finally:
        for k_, v in old.items():
            moe.moe_set_option(k_, v)


def test_wait_limit_option_validation(moe):
    with pytest.raises(moe.MoeError):
        moe.moe_set_option(moe.MOE_OPT_WAIT_LIMIT_US, 0)
    with pytest.raises(moe.MoeError):
        moe.moe_set_option(moe.MOE_OPT_TEST_TIMEOUT, 2)
    assert moe.moe_get_option(moe.MOE_OPT_WAIT_LIMIT_US) >= 1
