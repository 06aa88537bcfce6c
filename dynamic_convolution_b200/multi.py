"""Multi-GPU plumbing: one process per GPU, independent batches per rank (the
method is per-sample, so the forward shards with no exchange on the data
path), the timing rule "the job takes as long as its slowest rank", and, for
data-parallel training, the one real exchange of the backward: the parameter
gradients (experts, their biases, the router's weight and bias) are sums over
samples, so each rank's sums over its own samples are added over all ranks."""
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


def allreduce_gradients(tensors, bucket_bytes: int = 64 << 20) -> None:
    """Sum each tensor over all ranks, in place (identity when
    torch.distributed is not initialised or has one rank). The tensors are the
    parameter gradients of one layer (dexperts, dbias, dWr, dbr from the
    backward calls), each a sum over this rank's samples; after the call every
    rank holds the sums over the whole batch. Same-dtype tensors are packed
    into flat buckets of at most `bucket_bytes` (fewer, larger collectives:
    NCCL on GPUs, gloo on CPUs) in the order given, so every rank issues the
    same collectives in the same order."""
    import torch
    import torch.distributed as dist
    ts = [t for t in tensors if t is not None and t.numel() > 0]
    if not ts or not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return
    bucket: list = []
    size = 0

    def flush():
        nonlocal bucket, size
        if not bucket:
            return
        flat = torch.cat([t.reshape(-1) for t in bucket])
        dist.all_reduce(flat, op=dist.ReduceOp.SUM)
        off = 0
        for t in bucket:
            n = t.numel()
            t.copy_(flat[off:off + n].view_as(t))
            off += n
        bucket, size = [], 0

    for t in ts:
        nbytes = t.numel() * t.element_size()
        if bucket and (t.dtype != bucket[0].dtype or size + nbytes > bucket_bytes):
            flush()
        bucket.append(t)
        size += nbytes
    flush()
