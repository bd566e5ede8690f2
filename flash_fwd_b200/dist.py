"""Process-group plumbing for running the attention path on several GPUs.

The path shards with no exchange step: every (batch, head) -- and in the
forward every query tile -- is independent, so N ranks either run N
independent replicas of a workload (weak scaling, what the benchmark does) or
split the batch-head units of one workload (shard_range) without any data-path
collective.  The only collectives here are the barrier and the max-over-ranks
reduction of timings.
"""
import datetime
import os

import torch
import torch.distributed as dist


def env_ranks():
    """(rank, world_size, local_rank) from the torchrun environment."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init(backend, timeout_s=120):
    rank, world, local = env_ranks()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, local


def barrier(device=None):
    if dist.is_initialized() and dist.get_world_size() > 1:
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index if device is not None else torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x, device=None):
    """The maximum of a float over all ranks (identity with one rank)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_range(n_units, world, rank):
    """Contiguous [lo, hi) share of n_units for this rank (sizes differ by <= 1)."""
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    hi = lo + base + (1 if rank < extra else 0)
    return lo, hi


def aggregate_throughput(work_per_rank, max_ms):
    """Whole-job throughput: all ranks' work divided by the slowest rank's time."""
    return sum(work_per_rank) / (max_ms / 1e3)


def shutdown():
    if dist.is_initialized():
        dist.destroy_process_group()
