"""Process-group plumbing for running the kernels on several GPUs of a node.

The per-token hot path shards without any data exchange: every token row
(and every head of it) is independent, so each rank processes its own
samples and nothing crosses NVLink on the data path.  The only collectives
are the timing ones: a barrier around the timed region and the max / sum
reductions that turn per-rank times and unit counts into one whole-job
throughput.  One process per GPU, launched by torchrun (RANK, LOCAL_RANK,
WORLD_SIZE, MASTER_ADDR/PORT from the environment); NCCL on GPUs, gloo for
the CPU tests.
"""
import datetime
import os
from typing import Tuple

import torch
import torch.distributed as dist


def env_world() -> Tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> Tuple[int, int, int]:
    """Join the process group if WORLD_SIZE > 1; returns (rank, local_rank, world)."""
    rank, local_rank, world = env_world()
    if world > 1 and not dist.is_initialized():
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend=backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    elif backend == "nccl" and torch.cuda.is_available():
        torch.cuda.set_device(local_rank)
    return rank, local_rank, world


def active() -> bool:
    return dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1


def _device():
    if active() and dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier() -> None:
    if active():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def _reduce(x: float, op) -> float:
    if not active():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float) -> float:
    return _reduce(x, dist.ReduceOp.MAX)


def sum_over_ranks(x: float) -> float:
    return _reduce(x, dist.ReduceOp.SUM)


def job_throughput(local_units: float, local_seconds: float) -> Tuple[float, float, float]:
    """Whole-job throughput: units of all ranks / the slowest rank's time.
    Returns (units_per_second, total_units, max_seconds)."""
    total = sum_over_ranks(local_units)
    slowest = max_over_ranks(local_seconds)
    return (total / slowest if slowest > 0 else 0.0), total, slowest


def shutdown() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
