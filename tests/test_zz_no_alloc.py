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


def test_sort_static_at_its_limits(moe):
    # the largest accepted call fills the whole array: T*k = 65536 pairs over
    # E = 1024 experts (64 chunk histograms of 1024 entries)
    idx = _idx(4096, 16, 1024, 4)
    ref = moe.moe_sort(idx, 1024)
    got = moe.moe_sort_static(idx, 1024)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


def test_sort_static_refuses_oversized_calls(moe):
    idx = torch.zeros((65536 // 6 + 1, 6), dtype=torch.int32, device="cuda")
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_sort_static(idx, 256)
    assert ei.value.status == -2
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_sort_static(torch.zeros((4, 2), dtype=torch.int32, device="cuda"), 1025)
    assert ei.value.status == -2


def test_sort_static_reports_bad_ids_in_offsets(moe):
    # a caller of this variant has no workspace to read an error word from:
    # offsets[E] counts the pairs sorted, so bad ids show as offsets[E] < T*k
    for T, k, E in [(6, 2, 4), (3000, 2, 8)]:
        idx = _idx(T, k, E, 5)
        idx[1, 1] = E + 3
        idx[T - 1, 0] = -1
        ref = moe.moe_sort(idx, E)
        got = moe.moe_sort_static(idx, E)
        torch.cuda.synchronize()
        assert int(got[2][E]) == T * k - 2
        assert torch.equal(got[2], ref[2])
