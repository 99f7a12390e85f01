"""The whole layer captured in a CUDA graph.

moe_layer_forward makes no host synchronisation and no allocation, and its
kernels are launched with programmatic dependent launch, so the call can be
captured once and replayed.  The layer is deterministic (exact partial sums,
fixed-order combine), so a replay must reproduce the eager call bit for bit,
also after new inputs are written into the captured buffers.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


def cu(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _case(name):
    if name == "decode_T8":
        w = synth.WORKLOADS[name]
        return w, synth.make(w), None
    # several experts with hundreds of rows: the tensor-core path (forced for
    # every expert), several token tiles per expert, ragged tails
    w = synth.custom("graph_tc", 300, 512, 4, 2, 256, 71)
    return w, synth.make(w), 1


@pytest.mark.parametrize("name", ["decode_T8", "tensor_core_T300"])
def test_layer_graph_replay_matches_eager(moe, name):
    w, d, tc_min = _case(name)
    old = moe.moe_get_option(moe.MOE_OPT_TC_MIN_ROWS)
    if tc_min is not None:
        moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, tc_min)
    try:
        T, H, I, E, k = w.T, w.H, w.I, w.E, w.k
        packed = moe.moe_pack_weights(cu(d["w1_codes"]), cu(d["w1_scales"]), cu(d["w2_codes"]),
                                      cu(d["w2_scales"]))
        logits = cu(d["logits"])
        x = cu(d["x"]).view(torch.bfloat16)
        ws = torch.zeros(moe.moe_layer_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device="cuda")
        y_eager = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
        y_graph = torch.empty_like(y_eager)

        moe.moe_layer_forward(logits, x, packed, H, I, E, k, ws=ws, y=y_eager)  # also warms up
        torch.cuda.synchronize()
        assert moe.moe_check_device_flag(ws) == 0

        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            moe.moe_layer_forward(logits, x, packed, H, I, E, k, ws=ws, y=y_graph)
        g.replay()
        torch.cuda.synchronize()
        assert moe.moe_check_device_flag(ws) == 0
        assert torch.equal(y_graph.view(torch.int16), y_eager.view(torch.int16))

        # new inputs through the same graph: reversed token order, negated logits
        x.copy_(torch.flip(x, dims=[0]))
        logits.copy_(-torch.flip(logits, dims=[0]))
        g.replay()
        torch.cuda.synchronize()
        y_eager2 = moe.moe_layer_forward(logits, x, packed, H, I, E, k, ws=torch.zeros_like(ws))
        torch.cuda.synchronize()
        assert torch.equal(y_graph.view(torch.int16), y_eager2.view(torch.int16))
        assert not torch.equal(y_eager2.view(torch.int16), y_eager.view(torch.int16))
        del g
    finally:
        moe.moe_set_option(moe.MOE_OPT_TC_MIN_ROWS, old)
