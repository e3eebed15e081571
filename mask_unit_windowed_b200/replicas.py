"""Host-side plumbing for running the backbone as independent replicas, one process per GPU.

Images are independent through the whole Hiera backbone ("Phase 4: Hiera Backbone MLX
Port", Architecture Summary: every stage works on one image's tokens), so a global batch
splits across ranks with no collective on the data path. What remains is bookkeeping:

- shard_images:        the contiguous slice of a global batch a rank processes;
- max_over_ranks:      the job's time is the slowest rank's (one all-reduce MAX of a
                       scalar, on whatever backend the process group uses);
- job_throughput:      units all ranks processed divided by that time;
- gather_features:     an optional all-gather of a rank's outputs, for a caller that wants
                       the whole batch's features on every rank (off the timed path).

Nothing here launches a kernel; it works with the gloo backend on CPU tensors as well as
with NCCL on CUDA tensors.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def shard_images(global_batch: int, world: int, rank: int) -> tuple[int, int]:
    """(first image, count) of rank's contiguous share; the first global_batch % world
    ranks take one extra image, so every image belongs to exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if global_batch < 0:
        raise ValueError("global_batch must be >= 0")
    base, extra = divmod(global_batch, world)
    count = base + (1 if rank < extra else 0)
    first = rank * base + min(rank, extra)
    return first, count


def max_over_ranks(value: float, device: torch.device | str = "cpu") -> float:
    """The maximum of a per-rank scalar over the default process group (the value itself
    when no group is initialised)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Units per second of the whole job: all ranks' units over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("max_ms must be > 0")
    return units_per_rank * world / (max_ms / 1000.0)


def gather_features(local: torch.Tensor, counts: list[int]) -> torch.Tensor:
    """All-gather of per-rank outputs [count_r, ...] (counts from shard_images, in rank
    order) into the global batch [sum(counts), ...] on every rank."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return local
    world = dist.get_world_size()
    if len(counts) != world or local.shape[0] != counts[dist.get_rank()]:
        raise ValueError("counts must hold every rank's batch share")
    width = max(counts)
    padded = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype,
                         device=local.device)
    padded[:local.shape[0]] = local
    parts = [torch.empty_like(padded) for _ in range(world)]
    dist.all_gather(parts, padded)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)
