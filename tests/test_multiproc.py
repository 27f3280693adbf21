"""Host-side multi-process logic of bench.py on CPU: two gloo ranks on 127.0.0.1.

The bench runs one process per GPU (replicas: every rank streams its own copy of
the workload, no data-path collective).  What needs several processes is the
bookkeeping: the barrier around the timed region, the max over ranks of the
device time, and the whole-job value.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world)
    d.init("gloo")
    d.barrier()
    ms = d.max(1.0 + rank, "cpu")   # rank r measured 1 + r ms; the job takes the slowest
    value = bench.whole_job_gbps(d.world, 1e9, ms)
    d.barrier()
    d.close()
    q.put((rank, d.world, ms, value))


def test_two_gloo_ranks_barrier_and_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, w, ms, value in res:
        assert w == world
        assert ms == 2.0                       # max over ranks
        assert value == pytest.approx(1000.0)  # 2 ranks x 1 GB in 2 ms


def test_whole_job_value_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_gbps(1, 35651584 * 16, 0.2)
    assert bench.whole_job_gbps(8, 35651584 * 16, 0.2) == pytest.approx(8 * one)


def test_reference_arm_other_ranks_do_no_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    d = bench.Dist(2)
    assert bench.run_reference(None, d) is None


def test_profiled_traffic_only_for_the_profiled_source(tmp_path, monkeypatch):
    """The roofline's DRAM traffic comes from a committed ncu summary only while the
    kernel source still hashes to the profiled one; otherwise it is reported as null."""
    import hashlib
    import json

    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    (tmp_path / "profiles").mkdir()
    entry = {"source": "k.cu", "source_sha256": hashlib.sha256(b"kernel v1").hexdigest(),
             "dram_bytes_per_launch": 123}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"k": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("k") == 123
    assert bench.profiled_traffic("other") is None
    src.write_text("kernel v2")
    assert bench.profiled_traffic("k") is None
