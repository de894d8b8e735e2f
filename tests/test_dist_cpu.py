"""The multi-process plumbing of bench.py on CPU: two ranks over gloo on
127.0.0.1 (the GPU path uses NCCL with the same calls). Weak-scaling replicas:
each rank runs its own copy of the workload, the timing reduction takes the
slowest rank, and the job's value counts every rank's work."""
from __future__ import annotations

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    w, r, loc = bench.dist_setup(world, backend="gloo")
    bench.barrier(w)
    slowest = bench.max_over_ranks(10.0 + rank, w)  # rank 1 is the slow one
    value = bench.job_tflops(2e12, slowest, w)
    ref = bench.run_reference(type("A", (), {"workload": 1, "warmup": 0, "steps": 0})()) if r == 1 else "skipped"
    bench.barrier(w)
    dist.destroy_process_group()
    q.put((r, w, loc, slowest, value, ref))


def test_two_rank_replicas_over_gloo():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, w, loc, slowest, value, ref) in enumerate(res):
        assert (r, w, loc) == (rank, 2, rank)
        assert slowest == 11.0                      # the max over ranks, on every rank
        assert value == pytest.approx(2 * 2e12 / 11e-3 / 1e12)  # both ranks' work / the slowest time
    assert res[1][5] is None                        # the oracle arm runs on rank 0 only


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tflops(1e12, 1.0, 1) == pytest.approx(1000.0)
