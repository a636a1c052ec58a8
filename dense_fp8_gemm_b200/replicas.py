"""Independent replicas over several GPUs (one process per GPU).

The Spense GEMM has no exchange step: every rank runs the same workload on its
own GPU. The only cross-rank operations are a barrier around the timed region
and the max-over-ranks of the measured times, so the whole job's throughput is
(units every rank processed) / (slowest rank's time). These helpers hold that
logic so it can be tested with the gloo backend on CPU.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankInfo:
    world: int
    rank: int
    local: int


def from_env() -> RankInfo:
    """Rank layout from the torchrun environment (1 process when absent)."""
    return RankInfo(int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(info: RankInfo, backend: str, timeout_s: float = 120.0, device=None):
    """Join the process group when there is more than one rank (short timeout,
    so ranks that wait for a missing peer fail instead of hanging). `device`
    (a torch.device, for NCCL) binds the group to this rank's GPU."""
    if info.world <= 1:
        return None
    import torch.distributed as dist
    kw = {} if device is None else {"device_id": device}
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return dist


def barrier(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(info: RankInfo, values, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks."""
    values = [float(v) for v in values]
    if info.world <= 1:
        return values
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_rate(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput: every rank processed `units_per_rank` units; the
    job took as long as its slowest rank."""
    return units_per_rank * world / slowest_seconds


def finalize(info: RankInfo):
    if info.world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
