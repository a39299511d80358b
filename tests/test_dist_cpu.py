"""Multi-rank plumbing of bench.py on CPU processes (gloo, world size 2): the
barrier, the max-over-ranks job time, weak-scaling throughput, per-rank
sequences, and the reference arm running on rank 0 only.  No GPU is used:
the data path has no collective (every rank decodes its own sequence), so the
host-side logic is all there is to cover."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank), CSA2_DIST_BACKEND="gloo")
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(world)
    try:
        bench.barrier(w)
        # rank r took 10 + 5 r ms: the job's time is the slowest rank's
        ms = bench.max_over_ranks(10.0 + 5.0 * r, w)
        value = bench.job_throughput(w, 8, 100, ms)
        seed = bench.rank_seed(7, r)

        class A:   # the reference arm's arguments (rank 0 only does work)
            workload, seed, ref_budget, steps, warmup = "tiny4k", 0, 0.5, 1, 1
        ran = None
        if r != 0:
            ran = bench.run_reference(A, w, r) is None
        bench.barrier(w)
        out.put((r, w, ms, value, seed, ran))
    finally:
        dist.destroy_process_group()


def test_two_rank_plumbing():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, ms0, v0, s0, _), (r1, w1, ms1, v1, s1, ran1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert ms0 == ms1 == 15.0                           # max over ranks, seen by both
    assert v0 == v1 == pytest.approx(2 * 8 * 100 / 0.015)   # whole-job layer executions per second
    assert (s0, s1) == (7, 8)                           # independent sequences per rank
    assert ran1 is True                                 # the reference arm returns at once off rank 0
