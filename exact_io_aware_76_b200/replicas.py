"""Host-side logic for running the attention path as independent replicas, one process per GPU.

Every (batch, head, query tile) of exact attention is independent and the forward needs no exchange, so N GPUs
run N independent problems (weak scaling) and no collective touches the data path. The process group is used
only to line the ranks up before and after a timed region and to take the maximum of their device times.
"""
import datetime
import os

import torch
import torch.distributed as dist


def env_rank():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


def init(backend, timeout_s=120):
    """Join the process group described by the torchrun environment (no-op for a single process)."""
    rank, world, _ = env_rank()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def barrier(device=None):
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value, device=None):
    """Maximum of a float over all ranks (the value itself for a single process)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base_seed, rank):
    """Each replica draws its own synthetic problem."""
    return int(base_seed) + 7919 * int(rank)


def shard(n_units, rank, world):
    """Contiguous split of n_units independent units over the ranks (sizes differ by at most one)."""
    q, r = divmod(int(n_units), int(world))
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def shutdown():
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
