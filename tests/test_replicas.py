"""Replica plumbing on CPU: two gloo ranks (world size 2) exercising the host-side logic the
multi-GPU bench and a multi-GPU caller use. The backbone itself needs no collective
(images are independent), so this covers the sharding of a batch, the max-over-ranks time,
the job throughput and the optional feature all-gather."""

import os
import socket
import tempfile

import pytest
import torch
import torch.multiprocessing as mp

from mask_unit_windowed_b200 import replicas


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir, global_batch):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        first, count = replicas.shard_images(global_batch, world, rank)
        counts = [replicas.shard_images(global_batch, world, r)[1] for r in range(world)]
        # a rank's "features": its images' global indices, so the gather is checkable
        local = torch.arange(first, first + count, dtype=torch.float32)[:, None].repeat(1, 3)
        gathered = replicas.gather_features(local, counts)
        per_rank_ms = 10.0 + 5.0 * rank
        mx = replicas.max_over_ranks(per_rank_ms)
        thr = replicas.job_throughput(count, world, mx)
        torch.save({"first": first, "count": count, "gathered": gathered, "max_ms": mx,
                    "thr": thr}, os.path.join(out_dir, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("global_batch", [8, 7])
def test_two_gloo_ranks(global_batch):
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_worker, args=(world, _free_port(), d, global_batch), nprocs=world,
                           join=True, start_method="spawn")
        res = [torch.load(os.path.join(d, f"r{r}.pt")) for r in range(world)]
    # shards partition the batch, contiguous and in rank order
    assert res[0]["first"] == 0
    assert res[0]["first"] + res[0]["count"] == res[1]["first"]
    assert res[1]["first"] + res[1]["count"] == global_batch
    # every rank sees the slowest rank's time
    assert all(r["max_ms"] == 15.0 for r in res)
    # the gather returns the whole batch in order on every rank
    want = torch.arange(global_batch, dtype=torch.float32)[:, None].repeat(1, 3)
    for r in res:
        assert torch.equal(r["gathered"], want)
    # throughput: all ranks' units over the slowest time (equal shares when it divides)
    if global_batch % world == 0:
        assert all(abs(r["thr"] - global_batch / 0.015) < 1e-6 for r in res)


def test_shard_images_edge_cases():
    assert replicas.shard_images(0, 4, 3) == (0, 0)
    assert [replicas.shard_images(5, 3, r) for r in range(3)] == [(0, 2), (2, 2), (4, 1)]
    assert replicas.shard_images(3, 8, 7) == (3, 0)
    with pytest.raises(ValueError):
        replicas.shard_images(4, 2, 2)
    with pytest.raises(ValueError):
        replicas.job_throughput(1, 1, 0.0)
    # without a process group the helpers are the identity
    assert replicas.max_over_ranks(3.5) == 3.5
    t = torch.ones(2, 2)
    assert replicas.gather_features(t, [2]) is t
