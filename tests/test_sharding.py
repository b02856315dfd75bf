"""Multi-rank host logic on CPU: two gloo ranks shard a batch and gather it.

The attention call itself is replaced by a stand-in (the shard step must
not care what runs on each slice); the CUDA path is covered by the GPU tests.
"""
import os

import pytest
import torch
import torch.multiprocessing as mp

from masked_grouped_query_b200.sharding import attention_shard, gather_outputs, shard_batch


@pytest.mark.parametrize("batch,world", [(0, 2), (1, 2), (5, 2), (16, 3), (7, 8)])
def test_shard_batch_covers_every_row_once(batch, world):
    seen = []
    for r in range(world):
        s, c = shard_batch(batch, r, world)
        seen.extend(range(s, s + c))
    assert seen == list(range(batch))
    counts = [shard_batch(batch, r, world)[1] for r in range(world)]
    assert max(counts) - min(counts) <= 1


def test_shard_batch_rejects_bad_ranks():
    with pytest.raises(ValueError):
        shard_batch(4, 2, 2)
    with pytest.raises(ValueError):
        shard_batch(4, 0, 0)


def _stand_in(q, k, v, **kw):
    # shape of attention's output (q's), depends on k and v of the same rows
    return q * 2 + k.mean(dim=(1, 2), keepdim=True) + v.sum(dim=(1, 2), keepdim=True)


def _worker(rank, world, port, batch, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(7)
        q = torch.randn(batch, 4, 3, 8, generator=g)
        k = torch.randn(batch, 2, 5, 8, generator=g)
        v = torch.randn(batch, 2, 5, 8, generator=g)
        local = attention_shard(q, k, v, rank, world, _stand_in)
        full = gather_outputs(local, batch)
        want = _stand_in(q, k, v)
        assert torch.equal(full, want), "gathered output differs"
        if rank == 0:
            torch.save(full, result_path)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("batch", [5, 2, 1])
def test_two_gloo_ranks_shard_and_gather(batch, tmp_path):
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    out = tmp_path / "full.pt"
    mp.spawn(_worker, args=(2, port, batch, str(out)), nprocs=2, join=True)
    assert torch.load(out).shape[0] == batch
