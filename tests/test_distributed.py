"""Multi-process plumbing of bench.py on CPU: world size 2 over gloo.

The layer runs on one GPU per rank with no data exchange (replicas); what the
ranks share is the barrier around the timed region, the max-over-ranks time and
the whole-job throughput.  These run without a GPU.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist, r, w, local = bench.dist_setup(backend="gloo")
    try:
        bench.barrier(dist)
        t = bench.max_over_ranks(dist, 10.0 + 5.0 * r)   # rank 1 is the slower one
        v = bench.whole_job_gbs(1_000_000, 100, w, t)
        out.put((r, w, local, t, v))
        bench.barrier(dist)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_max_and_whole_job_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    for r, w, local, t, v in res:
        assert local == r
        assert t == 15.0                      # max over ranks, seen by both
        assert v == pytest.approx(2 * 1_000_000 * 100 / 15e-3 / 1e9)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    old = os.environ.pop("WORLD_SIZE", None)
    try:
        dist, r, w, local = bench.dist_setup(backend="gloo")
        assert dist is None and (r, w, local) == (0, 1, 0)
        assert bench.max_over_ranks(None, 3.5) == 3.5
    finally:
        if old is not None:
            os.environ["WORLD_SIZE"] = old


def test_reference_arm_other_ranks_do_nothing(capsys):
    sys.path.insert(0, ROOT)
    import bench
    old = os.environ.get("RANK")
    os.environ["RANK"] = "1"
    try:
        args = bench.argparse.Namespace(workload="tiny", steps=3, warmup=3, gpus=2)
        bench.run_reference(args)
        assert capsys.readouterr().out == ""
    finally:
        if old is None:
            del os.environ["RANK"]
        else:
            os.environ["RANK"] = old
