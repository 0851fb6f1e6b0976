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


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
