"""Multi-rank replica logic on CPU: two gloo ranks on 127.0.0.1.

The GEMM has no exchange step, so running on N GPUs means N independent
replicas; what crosses ranks is the barrier and the max-over-ranks timing.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

from dense_fp8_gemm_b200 import replicas


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    info = replicas.from_env()
    replicas.init(info, "gloo", timeout_s=30)
    replicas.barrier(info)
    # each rank "measured" a different time; rank 1 is the slowest
    times = [1.0 + rank, 0.5 * (rank + 1)]
    tmax = replicas.max_over_ranks(info, times)
    rate = replicas.job_rate(units_per_rank=100.0, world=info.world, slowest_seconds=tmax[0])
    out.put((rank, tmax, rate))
    replicas.finalize(info)


def test_two_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=60) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, tmax, rate in res:
        assert tmax == [2.0, 1.0]  # max over ranks, element-wise
        assert rate == pytest.approx(100.0 * 2 / 2.0)


def test_single_rank_needs_no_process_group():
    info = replicas.RankInfo(1, 0, 0)
    assert replicas.init(info, "gloo") is None
    assert replicas.max_over_ranks(info, [3.0]) == [3.0]
    assert replicas.job_rate(10.0, 1, 2.0) == 5.0
