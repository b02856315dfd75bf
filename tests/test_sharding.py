"""Multi-rank host logic on CPU: gloo ranks shard (batch, kv head) units and
gather the outputs.

Each rank's attention is the fp64 oracle itself on its sub-problem (batch =
its unit count, the group's q heads, one kv head), so the gathered output
must equal the oracle on the whole problem, element for element; the CUDA
path is covered by the GPU tests.
"""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from masked_grouped_query_b200.inputs import Workload, make_inputs
from masked_grouped_query_b200.sharding import (attention_shard, gather_outputs, shard_batch,
                                                shard_range, unit_views)


@pytest.mark.parametrize("n,world", [(0, 2), (1, 2), (5, 2), (16, 3), (7, 8), (3, 2)])
def test_shard_range_covers_every_item_once(n, world):
    seen = []
    for r in range(world):
        s, c = shard_range(n, r, world)
        seen.extend(range(s, s + c))
    assert seen == list(range(n))
    counts = [shard_range(n, r, world)[1] for r in range(world)]
    assert max(counts) - min(counts) <= 1
    assert [shard_batch(n, r, world) for r in range(world)] == \
        [shard_range(n, r, world) for r in range(world)]


def test_shard_range_rejects_bad_ranks():
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)
    with pytest.raises(ValueError):
        shard_range(4, 0, 0)


def test_unit_views_share_memory_and_order():
    # unit u = (b, kv head) = divmod(u, Hkv); its q rows are heads
    # [kvh * g, (kvh + 1) * g) of batch row b.
    q = torch.arange(2 * 6 * 3 * 8, dtype=torch.float32).reshape(2, 6, 3, 8)
    k = torch.arange(2 * 3 * 5 * 8, dtype=torch.float32).reshape(2, 3, 5, 8)
    qu, ku, vu = unit_views(q, k, k)
    assert qu.data_ptr() == q.data_ptr() and ku.data_ptr() == k.data_ptr()
    assert qu.shape == (6, 2, 3, 8) and ku.shape == (6, 1, 5, 8)
    for u in range(6):
        b, h = divmod(u, 3)
        assert torch.equal(qu[u], q[b, 2 * h:2 * h + 2])
        assert torch.equal(ku[u, 0], k[b, h])


def _oracle_fn(w):
    from oracle import oracle

    def fn(q, k, v):
        return torch.from_numpy(oracle.attention(q, k, v, causal=w.causal, window=w.window,
                                                 softcap=w.softcap))
    return fn


def _worker(rank, world, port, w, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        q, k, v = make_inputs(w)
        local = attention_shard(q, k, v, rank, world, _oracle_fn(w))
        full = gather_outputs(local, tuple(q.shape), w.num_kv_heads)
        if rank == 0:
            torch.save(full, result_path)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("w", [
    Workload("uneven_units", 1, 5, 40, 6, 3, 16, True, 9, 20.0, 3),    # 3 units on 2 ranks
    Workload("batch_and_heads", 5, 4, 33, 4, 2, 8, True, None, None, 4),   # 10 units
    Workload("one_unit", 1, 3, 17, 2, 1, 8, False, None, None, 5),     # rank 1 holds nothing
])
def test_two_gloo_ranks_equal_the_oracle_on_the_whole_problem(w, tmp_path):
    import socket

    from oracle import oracle
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    out = tmp_path / "full.pt"
    mp.spawn(_worker, args=(2, port, w, str(out)), nprocs=2, join=True)
    got = torch.load(out).numpy()
    q, k, v = make_inputs(w)
    want = oracle.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap)
    assert got.shape == want.shape
    assert np.array_equal(got, want)
