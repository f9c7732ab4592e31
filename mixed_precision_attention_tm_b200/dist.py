"""Host-side multi-rank plumbing of the benchmark (one process per GPU).

Tile-routed prefill partitions into independent (sequence, query tile, head)
units with no exchange between them, so ranks never communicate on the data
path: each rank processes its own independently seeded batch (weak scaling)
and the process group is used only to line the ranks up and to take the
maximum step time over ranks.
"""

from __future__ import annotations

import os

import torch


def world_info():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: distinct per rank, base seed on rank 0."""
    return int(base_seed) + 1000 * int(rank)


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def max_over_ranks(values, device="cpu"):
    """Element-wise maximum of a list of floats over all ranks (identity on
    one rank)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() \
            and torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(world: int, work_per_rank_step: float, ms_per_step: float, scale: float = 1e12) -> float:
    """Whole-job rate: the work of all ranks divided by the slowest rank's
    step time (ms), in units of `scale` per second."""
    return world * work_per_rank_step / (ms_per_step * 1e-3) / scale
