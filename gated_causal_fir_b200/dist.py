"""Multi-rank plumbing for replicas of the forward pass (one process per GPU).

The gated causal FIR shards with no exchange: sequences (and channel groups) are independent,
so N ranks each run the full kernel on their own batch.  Nothing here touches the data path;
it only sets up the process group, derives each rank's seed and batch slice, and reduces the
ranks' timings (max over ranks) on the host side of the timed region.
"""
import datetime
import os

import torch
import torch.distributed as dist


def env_world():
    """(rank, local_rank, world_size) from the torchrun environment (defaults: one process)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0):
    """Join the process group if WORLD_SIZE > 1; returns (rank, local_rank, world_size)."""
    rank, local_rank, world = env_world()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        kwargs = dict(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
        if backend == "nccl":
            kwargs["device_id"] = torch.device("cuda", local_rank)
        dist.init_process_group(**kwargs)
    return rank, local_rank, world


def barrier():
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest of every rank's value (identity with one process)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Distinct, reproducible input seed of each replica."""
    return base + 7919 * rank


def shard(n: int, rank: int, world: int):
    """[start, stop) of rank's share of n independent units (sizes differ by at most one)."""
    per, rem = divmod(n, world)
    start = rank * per + min(rank, rem)
    return start, start + per + (1 if rank < rem else 0)


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()
