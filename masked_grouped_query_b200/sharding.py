"""Splitting one attention call over the ranks of a process group.

The work partitions into independent (batch, kv head) units with no data
exchange, so a multi-GPU run needs no collective on the hot path: each rank
takes a contiguous slice of the batch (all kv heads of those batch rows, so
its q, k, v, o slices stay contiguous) and calls the CUDA path on it.  If the
caller wants the full output on every rank, ``gather_outputs`` does one
``all_gather`` (NCCL over NVLink on GPUs) after the kernels.
"""
from __future__ import annotations

import torch


def shard_batch(batch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, start + count) batch rows owned by ``rank``.

    The first ``batch % world`` ranks take one extra row; every row is owned
    by exactly one rank; ranks past the end get an empty slice.
    """
    if world < 1 or not 0 <= rank < world or batch < 0:
        raise ValueError("need 0 <= rank < world and batch >= 0")
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return start, count


def attention_shard(q, k, v, rank: int, world: int, attn_fn, **kwargs):
    """This rank's output rows: ``attn_fn`` on its batch slice of q, k, v."""
    start, count = shard_batch(q.shape[0], rank, world)
    sl = slice(start, start + count)
    return attn_fn(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), **kwargs)


def gather_outputs(local: torch.Tensor, batch: int, group=None) -> torch.Tensor:
    """All ranks' output slices concatenated along the batch (one all_gather).

    Slices may differ by one row; they are padded to the largest, gathered
    and trimmed back, so every rank ends with the full (batch, ...) output.
    """
    import torch.distributed as dist

    world = dist.get_world_size(group)
    counts = [shard_batch(batch, r, world)[1] for r in range(world)]
    width = max(counts) if counts else 0
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)
