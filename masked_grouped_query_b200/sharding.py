"""Splitting one attention call over the ranks of a process group.

The work partitions into independent (batch, kv head) units with no data
exchange: a unit owns the q rows of its GQA group's heads, its kv head's K
and V, and the matching output rows.  With q and o viewed as
[batch * num_kv_heads][group][q_len][head_dim] and k, v as
[batch * num_kv_heads][1][kv_len][head_dim], the units of a contiguous range
are contiguous slabs of all four tensors, so a rank's share is a plain view
(no copy): one sub-problem with batch = its unit count, group q heads and
one kv head, run through the CUDA path as is.  A multi-GPU run needs no
collective on the hot path; if the caller wants the full output on every
rank, ``gather_outputs`` does one ``all_gather`` (NCCL over NVLink on GPUs)
after the kernels.
"""
from __future__ import annotations

import torch


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous [start, start + count) of ``n`` items owned by ``rank``.

    The first ``n % world`` ranks take one extra item; every item is owned
    by exactly one rank; ranks past the end get an empty slice.
    """
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("need 0 <= rank < world and n >= 0")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return start, count


def shard_batch(batch: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous batch rows owned by ``rank`` (see ``shard_range``)."""
    return shard_range(batch, rank, world)


def unit_views(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    """q, k, v as (batch * kv heads) units: q [U][group][Lq][D], k and v
    [U][1][Lk][D] -- views of the same memory."""
    b, hq, lq, d = q.shape
    hkv, lk = k.shape[1], k.shape[2]
    if hq % hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    g = hq // hkv
    return (q.reshape(b * hkv, g, lq, d), k.reshape(b * hkv, 1, lk, d),
            v.reshape(b * hkv, 1, lk, d))


def attention_shard(q, k, v, rank: int, world: int, attn_fn, **kwargs):
    """This rank's units: ``attn_fn`` on its contiguous (batch, kv head)
    range, as a sub-problem with batch = its unit count, group q heads and
    one kv head.  Returns its output units [count][group][Lq][D]."""
    qu, ku, vu = unit_views(q, k, v)
    start, count = shard_range(qu.shape[0], rank, world)
    sl = slice(start, start + count)
    return attn_fn(qu[sl], ku[sl], vu[sl], **kwargs)


def gather_outputs(local: torch.Tensor, q_shape, num_kv_heads: int, group=None) -> torch.Tensor:
    """All ranks' output units concatenated and viewed with q's shape (one
    all_gather).  Slices may differ by one unit; they are padded to the
    largest, gathered and trimmed back, so every rank ends with the full
    (batch, num_q_heads, q_len, head_dim) output."""
    import torch.distributed as dist

    b, hq, lq, d = q_shape
    units = b * num_kv_heads
    world = dist.get_world_size(group)
    counts = [shard_range(units, r, world)[1] for r in range(world)]
    width = max(counts) if counts else 0
    pad = torch.zeros((width,) + tuple(local.shape[1:]), dtype=local.dtype,
                      device=local.device)
    pad[: local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    full = torch.cat([p[:c] for p, c in zip(parts, counts)], dim=0)
    return full.reshape(b, hq, lq, d)
