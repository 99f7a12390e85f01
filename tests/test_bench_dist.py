"""bench.py's multi-process plumbing on CPU: two gloo ranks.

The layer shards as independent replicas (one per GPU, no data-path
collective); what crosses ranks is only the timing: a barrier on both sides of
the timed region and the maximum of the ranks' device times, from which the
whole-job throughput is computed.  These run on the CPU with the gloo backend.
"""
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    return b


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    b = _bench()
    d = b.Dist(world, backend="gloo", device="cpu")
    d.barrier()
    ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    m = d.max(ms)
    d.barrier()
    q.put((rank, d.world, m, b.whole_job_value(d.world, 8, 100, m)))
    d.close()


def test_two_gloo_ranks_agree_on_max_time_and_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, m, v in res:
        assert w == world
        assert m == 15.0                       # every rank sees the slowest rank's time
        assert v == pytest.approx(2 * 8 * 100 / 15e-3)


def test_whole_job_value_is_weak_scaling():
    b = _bench()
    assert b.whole_job_value(1, 8, 1000, 200.0) == pytest.approx(40000.0)
    # twice the replicas in the same time: twice the tokens/s
    assert b.whole_job_value(2, 8, 1000, 200.0) == pytest.approx(80000.0)


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    # a summary gives its traffic only while its recorded hash matches the kernel
    # source; after a kernel change (before a new capture) it gives None
    import bench
    assert bench.profiled_traffic("no_such_summary.md") is None
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "kernel.cu"
    src.write_text("// a kernel\n")
    import hashlib
    good = hashlib.sha256(src.read_bytes()).hexdigest()
    (prof / "ok.md").write_text(f"    kernel_source: kernel.cu\n    kernel_source_sha256: {good}\n"
                                "    dram_bytes_per_launch: 1234\n")
    (prof / "stale.md").write_text(f"    kernel_source: kernel.cu\n    kernel_source_sha256: {'0' * 64}\n"
                                   "    dram_bytes_per_launch: 1234\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("ok.md") == 1234
    assert bench.profiled_traffic("stale.md") is None
