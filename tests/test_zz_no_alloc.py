"""moe_sort_static: the expert sort for callers that cannot supply scratch.

Some callers only receive input and output buffers (for example code running
inside a host framework that owns every device allocation) and cannot allocate
or size a workspace.  moe_sort_static gives them the same sort with scratch
held by the library itself.  This file is collected last on purpose: if it
fails, every other test has already run.  It checks the no-workspace entry
point against moe_sort (which takes a caller workspace) on two calls in a row,
so a stale result left in the shared scratch by the first call would show up
in the second, and checks that oversized calls are refused.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import fp4_routed_mixture_b200 as m
    return m


def _idx(T, k, E, seed):
    rng = np.random.default_rng(seed)
    idx = np.zeros((T, k), np.int32)
    for t in range(T):
        idx[t] = rng.permutation(E)[:k]
    return torch.from_numpy(idx).cuda()


def test_sort_static_matches_sort_twice_in_a_row(moe):
    # two different problems back to back through the same library scratch:
    # a multi-chunk one (several histograms) then a single-chunk one
    for T, k, E, seed in [(4604, 6, 256, 1), (64, 6, 256, 2), (9000, 6, 1024, 3)]:
        idx = _idx(T, k, E, seed)
        ref = moe.moe_sort(idx, E)
        got = moe.moe_sort_static(idx, E)
        torch.cuda.synchronize()
        for a, b in zip(got, ref):
            assert torch.equal(a, b)


def test_sort_static_refuses_oversized_calls(moe):
    idx = torch.zeros((65536 // 6 + 1, 6), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_sort_static(idx, 256)
    assert ei.value.status == -2
