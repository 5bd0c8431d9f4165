"""The multi-GPU host logic of bench.py on two gloo ranks (CPU, no GPU).

Each rank runs its own problem (weak scaling, no collective on the data path); the only
collective is the max of the per-rank step times, from which the whole-job throughput is
computed.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import datetime
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = bench.rank_workload(W.WORKLOADS["express32k"], rank)
        step_ms = [2.0, 3.5][rank]
        ms = bench.max_over_ranks(step_ms, dist, torch.device("cpu"))
        val = bench.job_value(world, w.B * w.H * w.T, ms)
        q.put((rank, w.data_seed, ms, val))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_host_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=5) for _ in range(2))
    seeds = {r[1] for r in res}
    assert len(seeds) == 2                                 # independent problems per rank
    assert all(r[2] == 3.5 for r in res)                   # the slowest rank bounds the job
    tokens = 32 * 32768
    assert all(abs(r[3] - 2 * tokens / 3.5e-3) < 1e-6 * r[3] for r in res)


def test_single_process_needs_no_collective():
    import bench
    assert bench.max_over_ranks(4.25, None, torch.device("cpu")) == 4.25
    assert bench.rank_workload(W.WORKLOADS["tiny"], 0) == W.WORKLOADS["tiny"]
