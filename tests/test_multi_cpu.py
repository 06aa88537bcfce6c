"""Multi-process (gloo, CPU) checks of the benchmark's multi-GPU plumbing:
max-over-ranks timing and the weak-scaling aggregate."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from dynamic_convolution_b200 import multi


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        w, r, lr = multi.dist_env()
        assert (w, r, lr) == (world, rank, rank)
        # rank-dependent "timings": the slowest rank decides
        mx = multi.max_over_ranks([1.0 + rank, 10.0 - rank])
        lo, hi = multi.shard(10, world, rank)
        q.put((rank, mx, (lo, hi)))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_max_and_shard():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, mx, _ in res:
        assert mx == [2.0, 10.0]
    assert [sh for _, _, sh in res] == [(0, 5), (5, 10)]


def test_single_process_identity_and_rate():
    assert multi.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    assert multi.weak_scaling_rate(64, 4, 0.5) == 512.0
    with pytest.raises(ValueError):
        multi.weak_scaling_rate(1, 1, 0.0)


@pytest.mark.parametrize("total,world", [(10, 3), (7, 7), (0, 2), (64, 8)])
def test_shard_partitions(total, world):
    parts = [multi.shard(total, world, r) for r in range(world)]
    assert parts[0][0] == 0 and parts[-1][1] == total
    assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    sizes = [e - b for b, e in parts]
    assert max(sizes) - min(sizes) <= 1


def _grad_worker(rank, world, port, q):
    """Each rank: the oracle's backward of its shard of a small layer, then the
    parameter gradients summed over ranks with multi.allreduce_gradients."""
    import numpy as np

    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x, dy, E, alpha, bias, Wr = _grad_layer()
        lo, hi = multi.shard(x.shape[0], world, rank)
        g = oracle.backward(x[lo:hi], dy[lo:hi], E, alpha[lo:hi], bias, Wr, oracle.SOFTMAX, 1.5,
                            stride=1, pad=1)
        ts = [torch.from_numpy(np.ascontiguousarray(g[k])) for k in ("dexperts", "dbias", "dWr", "dbr")]
        multi.allreduce_gradients(ts, bucket_bytes=4096)   # small buckets: several collectives
        q.put((rank, [t.numpy() for t in ts]))
    finally:
        dist.destroy_process_group()


def _grad_layer():
    import numpy as np
    rng = np.random.default_rng(0)
    B, C, Co, H, W, n = 5, 4, 6, 5, 4, 3
    return (rng.standard_normal((B, H, W, C)), rng.standard_normal((B, H, W, Co)),
            rng.standard_normal((n, Co, 3, 3, C)), rng.uniform(0.1, 1, (B, n)),
            rng.standard_normal((n, Co)), rng.standard_normal((n, C)))


def test_two_rank_gloo_gradient_allreduce_equals_full_batch():
    """Data-parallel backward: the parameter gradients of two shards, summed over
    the ranks, equal those of the whole batch (the sums over samples only
    change order)."""
    import numpy as np

    import oracle
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_grad_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    x, dy, E, alpha, bias, Wr = _grad_layer()
    full = oracle.backward(x, dy, E, alpha, bias, Wr, oracle.SOFTMAX, 1.5, stride=1, pad=1)
    for _, got in res:
        for k, v in zip(("dexperts", "dbias", "dWr", "dbr"), got):
            np.testing.assert_allclose(v, full[k], rtol=1e-12, atol=1e-12)


def test_allreduce_gradients_single_process_identity():
    t = torch.arange(6, dtype=torch.float32)
    multi.allreduce_gradients([t, None])
    assert t.tolist() == [0, 1, 2, 3, 4, 5]
