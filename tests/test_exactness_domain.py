"""The exactness domain of the two grouped GEMMs, probed at its edge.

Every term of the expert dot products is an integer multiple u of half the
row's smallest weight scale.  The streaming GEMM sums each 32-input block in
int32 and the blocks in fp64, exact while a row's scale bytes span fewer than
about 28 binades; the tensor-core GEMM accumulates in fp32 (TMEM), exact while
every partial sum stays below 2^24 u.  Here every W1 row holds the largest
E2M1 codes of one sign (random magnitudes 0..6) and scale bytes alternating 122
and 110 across its 32-input blocks (12 binades), and the activations are
positive, so the tensor-core partial sums reach ~2^32 u: the fp32 accumulator
must round.
Expected: the streaming path stays bit-exact (codes, scales); the tensor-core
path's h codes may move by one step in a few places, and y stays within the
layer's tolerance.  The number of moved codes is recorded in the assertion
messages.
"""
import numpy as np
import pytest

import oracle
import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from tests.test_gpu_parity import cu, run_layer, y_check  # noqa: E402


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


def _extreme_inputs():
    T, H, E, k, I = 40, 1024, 1, 1, 128
    w = synth.custom("edge", T, H, E, k, I, 95)
    d = synth.make(w)
    d["w1_codes"] &= 0x77                                 # non-negative codes: magnitudes 0..6
    blk = np.arange(H // 32)
    d["w1_scales"][:] = np.where(blk % 2 == 0, 122, 110).astype(np.uint8)[None, None, :]
    x = np.abs(synth.bf16_to_f32(d["x"]))                 # positive activations
    d["x"] = (x.view(np.uint32) >> 16).astype(np.uint16)
    return w, d


@pytest.mark.parametrize("tc_min", [1, 1000])
def test_same_sign_extreme_rows(moe, tc_min):
    old = moe.moe_get_option(moe.MOE_OPT_TC_MIN_ROWS)
    moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, tc_min)
    try:
        w, d = _extreme_inputs()
        o = oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                           d["w2_scales"], w.k)
        r = run_layer(moe, d, w)
        assert np.array_equal(r["dbg"]["xq"].cpu().numpy(), o["xq"])
        hq = r["dbg"]["hq"].cpu().numpy()
        sh = r["dbg"]["sh"].cpu().numpy()
        moved = int((hq != o["hq"][o["perm"]]).sum())
        if tc_min > 1:
            # streaming GEMM: inside its exactness domain, bit-exact
            assert moved == 0 and np.array_equal(sh, o["sh"][o["perm"]])
        else:
            # tensor cores: fp32 accumulation rounds; codes move by at most one step
            assert np.abs(hq.astype(np.int32) - o["hq"][o["perm"]].astype(np.int32)).max() <= 1, moved
            assert moved <= hq.size // 100, moved
        y_check(r["y"], o["y"])
    finally:
        moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, old)
