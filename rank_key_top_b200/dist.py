"""Process-group plumbing for running decode steps on several GPUs.

The decode path splits into independent (sequence, kv head) units with no
exchange between them, so N GPUs run N independent replicas, each on its own
batch (weak scaling). The only collectives are the timing barrier and the
maximum over ranks of the measured device time; nothing on the data path.
One process per GPU, launched by torchrun (RANK / LOCAL_RANK / WORLD_SIZE /
MASTER_ADDR / MASTER_PORT from the environment).
"""
import datetime
import os

import torch
import torch.distributed as dist


def init_from_env(backend: str = "nccl", timeout_s: float = 120.0):
    """Returns (rank, world, local_rank); joins the process group if world > 1."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        kwargs = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kwargs["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kwargs)
    return rank, world, local


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest value of x over all ranks (every rank gets it)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own batch: a distinct, reproducible seed."""
    return base_seed + 7919 * rank


def aggregate_rate(units_per_rank: int, world: int, max_seconds: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / max_seconds


def finish(world: int) -> None:
    if world > 1 and dist.is_initialized():
        dist.destroy_process_group()
