"""The multi-GPU bench path on CPU: two gloo ranks, each scanning its own
batch (weak scaling, no collective on the data path); the job time is the
max over ranks and the throughput counts the units of all ranks."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import ssm_gen


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        job_ms = bench.max_over_ranks(local_ms, world, device="cpu")
        inp = ssm_gen.make_s6_inputs(1, 8, 16, 4, seed=bench.rank_seed(rank))
        q.put((rank, job_ms, float(inp.x.sum())))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_scan_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert res[0][1] == res[1][1] == 15.0
    assert res[0][2] != res[1][2]          # different data per rank
    # all units of both ranks over the job time
    assert bench.job_throughput(100.0, 2, 10, 15.0) == pytest.approx(100 * 2 * 10 / 15e-3)


class _CpuEvent:
    """Stands in for a CUDA event: host clock, elapsed time in ms."""

    def record(self):
        import time
        self.t = time.perf_counter()

    def elapsed_time(self, other):
        return (other.t - self.t) * 1e3


def _timed_worker(rank, world, port, q):
    """bench.run_timed on a gloo rank with the device step stubbed by a host
    sleep (rank 1 twice as slow), on this rank's own seeded batch."""
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = ssm_gen.make_s6_inputs(2, 8, 16, 4, seed=bench.rank_seed(rank))
        calls = []

        def step():
            calls.append(1)
            time.sleep(0.01 * (1 + rank))

        flushed = []
        step_ms, job_ms = bench.run_timed(step, flushed.append, 5, world, "cpu", _CpuEvent, lambda: None)
        units = inp.batch * inp.seqlen * inp.dim * inp.dstate
        value = bench.job_throughput(units, world, 5, job_ms)
        q.put((rank, len(calls), flushed, sum(step_ms), job_ms, value, float(inp.x.sum())))
    finally:
        dist.destroy_process_group()


def test_run_timed_on_two_gloo_ranks():
    """The bench's timed region across ranks: every rank runs and flushes
    each step, the job time is the slowest rank's sum, and the throughput
    counts both ranks' units over it; each rank scans its own batch."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_timed_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r in res:
        assert r[1] == 5 and r[2] == [0, 1, 2, 3, 4]
    slow = max(r[3] for r in res)
    assert res[0][4] == res[1][4] == pytest.approx(slow)
    assert res[1][3] > res[0][3]                      # rank 1 set the job time
    units = 2 * 8 * 16 * 4
    assert res[0][5] == pytest.approx(units * 2 * 5 / (slow * 1e-3))
    assert res[0][6] != res[1][6]


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
