"""KV-cache append and the decode step on a cache (argument marshalling only).

``kv_append`` writes L new tokens' keys and values into a key cache and a
value cache at slots [position, position + L) ("KV Cache Update at a
Position", TensorTonic): every batch row and kv head receives the new
vectors in order, converted to the cache dtype, and every other slot keeps
its contents; the return value is the new filled length position + L.

``decode_append`` appends the step's tokens and then attends q to the first
position + L slots of the caches in place, as ``attention`` would with
kv_len = position + L.

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


def _flags(cache: torch.Tensor, new: torch.Tensor, seq_major: bool, new_head_major: bool) -> int:
    if cache.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"caches must be float32 or bfloat16, got {cache.dtype}")
    if new.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"new keys/values must be float32 or bfloat16, got {new.dtype}")
    return ((CACHE_SEQ_MAJOR if seq_major else 0) | (CACHE_F32 if cache.dtype == torch.float32
                                                     else 0)
            | (NEW_BF16 if new.dtype == torch.bfloat16 else 0)
            | (NEW_HEAD_MAJOR if new_head_major else 0))


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
              new_head_major: bool = False, stream=None) -> int:
    """Write new_k/new_v into the caches at ``position`` in place; return position + L."""
    b, s, h, d, length = _geometry(k_cache, v_cache, new_k, new_v, seq_major, new_head_major)
    flags = _flags(k_cache, new_k, seq_major, new_head_major)
    out_len = ctypes.c_int(-1)
    with torch.cuda.device(k_cache.device):
        rc = _lib.load().gqa_attn_kv_append(
            k_cache.data_ptr(), v_cache.data_ptr(), new_k.data_ptr(), new_v.data_ptr(), b, s, h,
            d, int(position), length, flags, ctypes.byref(out_len), _stream_handle(stream))
    _lib.check(rc, "gqa_attn_kv_append")
    return out_len.value


def decode_append(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                  new_k: torch.Tensor, new_v: torch.Tensor, position: int, *,
                  seq_major: bool = True, new_head_major: bool = False, causal: bool = True,
                  window: int | None = None, softcap: float | None = None,
                  out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Append the step's L tokens at ``position``, then attend q (batch,
    num_q_heads, L, head_dim) to cache slots [0, position + L); bf16 caches."""
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
    flags = _flags(k_cache, new_k, seq_major, new_head_major)
    c, w, sc = _args(window, softcap, causal)
    with torch.cuda.device(q.device):
        rc = _lib.load().gqa_attn_decode_append(
            q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), new_k.data_ptr(),
            new_v.data_ptr(), out.data_ptr(), b, length, int(position), s, hq, h, d, flags, c,
            w, sc, _stream_handle(stream))
    _lib.check(rc, "gqa_attn_decode_append")
    return out
