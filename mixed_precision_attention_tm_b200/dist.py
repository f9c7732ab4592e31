"""Host-side multi-rank plumbing (one process per GPU).

Tile-routed prefill partitions into independent (sequence, query tile, head)
units with no exchange between them.  Two ways of using several GPUs follow:

* independent batches (the benchmark's default, weak scaling): each rank
  processes its own seeded batch, and the process group only lines the ranks
  up and takes the maximum step time over ranks;
* one problem split by query heads (strong scaling): rank r computes a block
  of consecutive query heads (``head_shards``), cut where needed at the
  boundaries of grouped-query KV heads (``kv_segments``), and one all-gather
  of equal-size output slices (``all_gather_heads``) followed by the
  library's interleaving copy gives every rank the whole output.
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


def head_shards(hq: int, world: int):
    """Blocks of consecutive query heads per rank, [(h0, h1)] * world: the
    first hq % world ranks take one head more than the others (attention costs
    the same per head, so this balances the work to within one head)."""
    if hq < 1 or world < 1:
        raise ValueError("hq and world must be positive")
    base, extra = divmod(hq, world)
    out, h = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((h, h + n))
        h += n
    return out


def kv_segments(h0: int, h1: int, group: int):
    """Split query heads [h0, h1) into runs that one attention call can take
    with the library's head map (query head h reads KV head h // (Hq / Hkv)):
    [(s0, s1, k0, k1)], query heads [s0, s1) over KV heads [k0, k1).  A run
    of whole GQA groups becomes one segment; a group cut by a shard boundary
    becomes a segment of its own with a single KV head."""
    if group < 1:
        raise ValueError("group must be positive")
    segs, h = [], h0
    while h < h1:
        hk = h // group
        if h % group == 0 and h + group <= h1:
            n = (h1 - h) // group
            segs.append((h, h + n * group, hk, hk + n))
            h += n * group
        else:
            e = min(h1, (hk + 1) * group)
            segs.append((h, e, hk, hk + 1))
            h = e
    return segs


def all_gather_heads(gathered, local, group=None):
    """Gather every rank's output slice: local [T, h_cap, d] (contiguous, the
    same shape on every rank) into gathered [world, T, h_cap, d].  One
    collective; NCCL's all-gather into one tensor where the backend has it."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        gathered[0].copy_(local)
        return gathered
    if torch.distributed.get_backend(group) == "nccl":
        torch.distributed.all_gather_into_tensor(gathered, local, group=group)
    else:
        torch.distributed.all_gather(list(gathered.unbind(0)), local, group=group)
    return gathered
