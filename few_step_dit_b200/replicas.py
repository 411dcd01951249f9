"""Multi-GPU runs as independent replicas.

The Flash path does not shard inside one clip without an exchange step
(attention is all-to-all over tokens), so N GPUs run N independent clips: one
process per GPU, each with its own input seed, no collective on the data path.
The only collectives are the barriers around the timed region and the max of
the per-rank times (weak scaling: total units / slowest rank).
"""

from __future__ import annotations

import datetime
import os

import torch


def env():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(world, backend="nccl", timeout_s=600):
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def shutdown(world):
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


def input_seed(base, rank):
    """Each replica samples its own clip."""
    return base + rank


def barrier(world, device):
    if device.type == "cuda":
        torch.cuda.synchronize(device)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


def max_over_ranks(x, world, device):
    """Max of a per-rank float over all ranks (the slowest replica)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank, world, max_seconds):
    """Whole-job throughput: all ranks' units over the slowest rank's time."""
    return world * units_per_rank / max_seconds
