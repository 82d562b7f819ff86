"""Multi-process host logic of the replica / sequence-sharded mode, on CPU with gloo."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from tree_verify_b200.replicas import max_over_ranks, shard_sequences


@pytest.mark.parametrize("batch,world", [(16, 2), (17, 4), (1, 2), (3, 8)])
def test_shards_partition_the_batch(batch, world):
    seen = []
    for r in range(world):
        a, b = shard_sequences(batch, r, world)
        assert 0 <= a <= b <= batch
        seen.extend(range(a, b))
    assert seen == list(range(batch))
    sizes = [shard_sequences(batch, r, world)[1] - shard_sequences(batch, r, world)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_bad_rank():
    with pytest.raises(ValueError):
        shard_sequences(4, 2, 2)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = max_over_ranks([1.0 + rank, 10.0 - rank], dist=dist)
        a, b = shard_sequences(16, rank, world)
        out[rank] = torch.tensor(got + [a, b], dtype=torch.float64)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world, port = 2, 29511
    out = torch.zeros((world, 4), dtype=torch.float64).share_memory_()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r, 0].item() == 2.0 and out[r, 1].item() == 10.0
    assert out[0, 2:].tolist() == [0, 8] and out[1, 2:].tolist() == [8, 16]


def test_max_over_ranks_without_group():
    assert max_over_ranks([3, 4]) == [3.0, 4.0]
