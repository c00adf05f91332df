"""Multi-GPU plumbing for the benchmark: the hot path has no exchange step
(every GEMM is an independent problem), so N GPUs run N independent
replicas and the only cross-rank operations are a barrier around the timed
region and the max-over-ranks of the measured time.  Backend-agnostic so the
logic runs under `gloo` on CPU in the tests and `nccl` on GPUs."""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_ranks():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, local_rank: int, timeout_s: int = 120):
    """Initializes the default process group (short timeout so that ranks that
    wait for a missing peer end with an error instead of hanging)."""
    kw = {}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local_rank)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier():
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (the slowest replica's time)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return world * units_per_rank / seconds_max
