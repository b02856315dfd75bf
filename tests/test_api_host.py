"""Argument checks of the Python entry points that run before any device
call (CPU): wrong types, shapes and placements raise with a message; nothing
falls back to a CPU computation."""
import pytest
import torch

import masked_grouped_query_b200 as mgq


def _qkv(device="cpu", dtype=torch.bfloat16):
    q = torch.zeros(1, 4, 3, 64, dtype=dtype, device=device)
    k = torch.zeros(1, 2, 5, 64, dtype=dtype, device=device)
    return q, k, k.clone()


def test_attention_rejects_host_tensors():
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="attention_host"):
        mgq.attention(q, k, v, causal=True)


@pytest.mark.parametrize("bad, exc", [
    (lambda q: q.float(), TypeError),                 # dtype
    (lambda q: q[0], ValueError),                     # 3-D
    (lambda q: q.transpose(2, 3), ValueError),        # not contiguous
    (lambda q: q.tolist(), TypeError),                # not a tensor
])
def test_attention_rejects_bad_q(bad, exc):
    q, k, v = _qkv()
    with pytest.raises(exc):
        mgq.attention(bad(q), k, v)


def test_make_attention_checks_shapes_against_cfg():
    cfg = dict(batch=1, q_len=3, kv_len=5, num_q_heads=4, num_kv_heads=2, head_dim=64,
               causal=True, window=None, softcap=None, seed=7, name="x")
    f = mgq.make_attention(cfg)
    q, k, v = _qkv()
    with pytest.raises(ValueError, match="do not match cfg"):
        f(q[:, :2], k, v)
    with pytest.raises(ValueError, match="do not match cfg"):
        f(q, k[:, :, :4], v)


def test_attention_host_rejects_bad_dtype():
    q, k, v = _qkv()
    with pytest.raises(TypeError):
        mgq.attention_host(q.float(), k, v)


def test_kv_cache_entry_points_reject_host_tensors():
    cache = torch.zeros(1, 16, 2, 64, dtype=torch.bfloat16)
    new = torch.zeros(1, 1, 2, 64)
    with pytest.raises(ValueError, match="CUDA"):
        mgq.kv_append(cache, cache.clone(), new, new.clone(), 0, seq_major=True)


def test_unknown_override_name():
    with pytest.raises(KeyError):
        mgq.set_override("prefill_clusters", 1)
