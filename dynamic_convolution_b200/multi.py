"""Multi-GPU plumbing for the benchmark: one process per GPU, independent
batches per rank (the method is per-sample, so the batch shards with no
exchange on the data path), and the timing rule "the job takes as long as its
slowest rank". Only torch.distributed collectives on scalars are used here."""
from __future__ import annotations

import os


def dist_env() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard(total: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous [begin, end) share of `total` independent units for `rank`."""
    if world <= 0 or not 0 <= rank < world or total < 0:
        raise ValueError("bad shard arguments")
    base, extra = divmod(total, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum of a list of floats over all ranks (identity if
    torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    vals = [float(v) for v in values]
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def weak_scaling_rate(units_per_rank: int, world: int, seconds_max: float) -> float:
    """Whole-job throughput: every rank processed `units_per_rank` units and the
    job lasted as long as its slowest rank."""
    if seconds_max <= 0:
        raise ValueError("non-positive time")
    return world * units_per_rank / seconds_max
