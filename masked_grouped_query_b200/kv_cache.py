"""KV-cache append and the decode step on a cache (argument marshalling only).

``kv_append`` writes L new tokens' keys and values into a key cache and a
value cache at slots [position, position + L) ("KV Cache Update at a
Position", TensorTonic): every batch row and kv head receives the new
vectors in order, converted to the cache dtype, and every other slot keeps
its contents; the return value is the new filled length position + L.

``decode_append`` appends the step's tokens and then attends q to the first
position + L slots of the caches in place, as ``attention`` would with
kv_len = position + L.

``attention_ring`` attends to keys and values kept in ring buffers: key j
of the kv_len-key sequence sits in slot j % slots ("CSA2 attention on
Metal", TensorFold pull request 1709, "What this changes": decode rows over
ring windows).  ``ring=True`` makes ``kv_append`` / ``decode_append`` write
token p to slot p % slots and attend the same way.

Layouts: ``seq_major=True`` caches are (batch, slots, kv_heads, head_dim), the
page's layout; ``seq_major=False`` caches are (batch, kv_heads, slots,
head_dim), the layout ``attention`` reads.  New keys and values are
(batch, L, kv_heads, head_dim) (the page's) or, with ``new_head_major=True``,
(batch, kv_heads, L, head_dim), in fp32 (the page's) or bf16.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from .attention import _args, _check_tensor, _stream_handle

CACHE_SEQ_MAJOR = 0x1
CACHE_F32 = 0x2
NEW_BF16 = 0x4
NEW_HEAD_MAJOR = 0x8
RING = 0x10


def _flags(cache: torch.Tensor, new: torch.Tensor, seq_major: bool, new_head_major: bool,
           ring: bool = False) -> int:
    if cache.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"caches must be float32 or bfloat16, got {cache.dtype}")
    if new.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"new keys/values must be float32 or bfloat16, got {new.dtype}")
    return ((CACHE_SEQ_MAJOR if seq_major else 0) | (CACHE_F32 if cache.dtype == torch.float32
                                                     else 0)
            | (NEW_BF16 if new.dtype == torch.bfloat16 else 0)
            | (NEW_HEAD_MAJOR if new_head_major else 0) | (RING if ring else 0))


def _geometry(k_cache, v_cache, new_k, new_v, seq_major, new_head_major):
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache), ("new_k", new_k), ("new_v", new_v)):
        if not isinstance(t, torch.Tensor) or t.dim() != 4:
            raise ValueError(f"{n} must be a 4-D torch.Tensor")
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CUDA tensor")
    if k_cache.shape != v_cache.shape or k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache and v_cache must share shape and dtype")
    if new_k.shape != new_v.shape or new_k.dtype != new_v.dtype:
        raise ValueError("new_k and new_v must share shape and dtype")
    if seq_major:
        b, s, h, d = k_cache.shape
    else:
        b, h, s, d = k_cache.shape
    if new_head_major:
        nb, nh, length, nd = new_k.shape
    else:
        nb, length, nh, nd = new_k.shape
    if (nb, nh, nd) != (b, h, d):
        raise ValueError(f"new tokens {tuple(new_k.shape)} do not match the caches "
                         f"{tuple(k_cache.shape)}")
    return b, s, h, d, length


def kv_append(k_cache: torch.Tensor, v_cache: torch.Tensor, new_k: torch.Tensor,
              new_v: torch.Tensor, position: int, *, seq_major: bool = True,
              new_head_major: bool = False, ring: bool = False, stream=None) -> int:
    """Write new_k/new_v into the caches at ``position`` in place (ring: at
    slots (position + l) % slots); return position + L."""
    b, s, h, d, length = _geometry(k_cache, v_cache, new_k, new_v, seq_major, new_head_major)
    flags = _flags(k_cache, new_k, seq_major, new_head_major, ring)
    out_len = ctypes.c_int(-1)
    with torch.cuda.device(k_cache.device):
        rc = _lib.load().gqa_attn_kv_append(
            k_cache.data_ptr(), v_cache.data_ptr(), new_k.data_ptr(), new_v.data_ptr(), b, s, h,
            d, int(position), length, flags, ctypes.byref(out_len), _stream_handle(stream))
    _lib.check(rc, "gqa_attn_kv_append")
    return out_len.value


def decode_append(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  new_k: torch.Tensor, new_v: torch.Tensor, position: int, *,
                  seq_major: bool = True, new_head_major: bool = False, ring: bool = False,
                  causal: bool = True, window: int | None = None, softcap: float | None = None,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Append the step's L tokens at ``position``, then attend q (batch,
    num_q_heads, L, head_dim) to the keys [0, position + L) -- cache slots
    [0, position + L), or with ``ring`` slot j % slots for key j; bf16."""
    _check_tensor("q", q)
    b, s, h, d, length = _geometry(k_cache, v_cache, new_k, new_v, seq_major, new_head_major)
    qb, hq, lq, qd = q.shape
    if (qb, lq, qd) != (b, length, d):
        raise ValueError(f"q {tuple(q.shape)} does not match the new tokens "
                         f"{tuple(new_k.shape)}")
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_tensor("out", out)
        if out.shape != q.shape:
            raise ValueError("out must match q's shape")
    flags = _flags(k_cache, new_k, seq_major, new_head_major, ring)
    c, w, sc = _args(window, softcap, causal)
    with torch.cuda.device(q.device):
        rc = _lib.load().gqa_attn_decode_append(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), new_k.data_ptr(),
            new_v.data_ptr(), out.data_ptr(), b, length, int(position), s, hq, h, d, flags, c,
            w, sc, _stream_handle(stream))
    _lib.check(rc, "gqa_attn_decode_append")
    return out


def attention_ring(q: torch.Tensor, k_ring: torch.Tensor, v_ring: torch.Tensor, kv_len: int, *,
                   seq_major: bool = False, causal: bool = True, window: int | None = None,
                   softcap: float | None = None, out: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """Masked GQA attention of q (batch, num_q_heads, q_len, head_dim) over a
    kv_len-key sequence whose key j sits in ring slot j % slots of k_ring /
    v_ring ((batch, kv_heads, slots, head_dim), or (batch, slots, kv_heads,
    head_dim) with ``seq_major``); bf16, CUDA tensors."""
    for n, t in (("q", q), ("k_ring", k_ring), ("v_ring", v_ring)):
        _check_tensor(n, t)
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor")
    if k_ring.shape != v_ring.shape:
        raise ValueError("k_ring and v_ring must share a shape")
    b, hq, lq, d = q.shape
    if seq_major:
        bk, slots, hkv, dk = k_ring.shape
    else:
        bk, hkv, slots, dk = k_ring.shape
    if bk != b or dk != d:
        raise ValueError(f"ring {tuple(k_ring.shape)} does not match q {tuple(q.shape)}")
    if out is None:
        out = torch.empty_like(q)
    c, w, sc = _args(window, softcap, causal)
    with torch.cuda.device(q.device):
        rc = _lib.load().gqa_attn_fwd_ring(
            q.data_ptr(), k_ring.data_ptr(), v_ring.data_ptr(), out.data_ptr(), b, lq,
            int(kv_len), slots, hq, hkv, d, CACHE_SEQ_MAJOR if seq_major else 0, c, w, sc,
            _stream_handle(stream))
    _lib.check(rc, "gqa_attn_fwd_ring")
    return out
