"""Attention over ring-buffer K/V (sliding-window decode stored circularly)
against the fp64 oracle (GPU).

Key j of the kv_len-key sequence sits in ring slot j % S.  The oracle sees
the keys in order, rebuilt from the ring by ``oracle.kv_cache.ring_sequence``
(keys older than kv_len - S are no longer stored: they are filled with large
values, which the window must hide).  Bar: the attention tolerance of
``test_parity``.
"""
import numpy as np
import pytest
import torch

import masked_grouped_query_b200 as mgq
from masked_grouped_query_b200 import _lib
from masked_grouped_query_b200.inputs import make_cache_inputs
from oracle import kv_cache as okv
from oracle import oracle

from .test_parity import assert_close

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def linear_from_ring(ring_page: torch.Tensor, kv_len: int) -> torch.Tensor:
    """(B, S, H, D) ring -> keys in order as (B, H, kv_len, D) bf16."""
    fill = int(bits(torch.tensor([3.0e4], dtype=torch.bfloat16))[0])
    seq = okv.ring_sequence(bits(ring_page), kv_len, fill=fill)
    return bf16(seq).transpose(1, 2).contiguous()


RING_CASES = [
    # (batch, q_len, kv_len, slots, hq, hkv, d, causal, window, softcap, seq_major)
    (4, 1, 10000, 4096, 32, 8, 128, True, 4096, None, False),   # wrapped, unaligned wrap
    (2, 4, 33000, 4160, 64, 4, 128, True, 4096, 30.0, True),    # 16:1, reach 4099 <= 4160
    (3, 1, 700, 1024, 16, 4, 64, True, 512, None, False),       # not wrapped yet
    (2, 2, 5000, 320, 8, 8, 256, True, 300, 20.0, False),       # head_dim 256
    (1, 3, 4096, 4096, 12, 4, 96, False, None, None, True),     # no window: exactly full
    (2, 1, 8191, 64, 4, 2, 64, True, 64, None, False),          # one-tile ring
    (1, 20, 3000, 512, 4, 1, 128, True, 100, None, False),      # 80 rows per kv head
]


@pytest.mark.parametrize("case", RING_CASES, ids=[str(c) for c in RING_CASES])
def test_ring_attention_matches_oracle(case):
    b, lq, kv_len, slots, hq, hkv, d, causal, window, cap, seq_major = case
    x = make_cache_inputs(b, slots, hkv, d, 0, seed=kv_len + slots, num_q_heads=hq)
    q = torch.randn(b, hq, lq, d, generator=torch.Generator().manual_seed(slots)).bfloat16()
    kr, vr = x["k_cache"], x["v_cache"]          # (B, S, H, D)
    k_lin, v_lin = linear_from_ring(kr, kv_len), linear_from_ring(vr, kv_len)
    want = oracle.attention(q, k_lin, v_lin, causal=causal, window=window, softcap=cap)
    kd = (kr if seq_major else kr.transpose(1, 2)).contiguous().cuda()
    vd = (vr if seq_major else vr.transpose(1, 2)).contiguous().cuda()
    got = mgq.attention_ring(q.cuda(), kd, vd, kv_len, seq_major=seq_major, causal=causal,
                             window=window, softcap=cap)
    torch.cuda.synchronize()
    assert_close(got, want, f"ring {case}")
    again = mgq.attention_ring(q.cuda(), kd, vd, kv_len, seq_major=seq_major, causal=causal,
                               window=window, softcap=cap)
    torch.cuda.synchronize()
    assert torch.equal(got, again)   # deterministic


def test_ring_too_small_is_rejected():
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16, device="cuda")
    ring = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16, device="cuda")
    for kw in (dict(window=128), dict(window=None)):
        with pytest.raises(_lib.GqaAttnError) as e:
            mgq.attention_ring(q, ring, ring, 1000, **kw)
        assert e.value.code == -12
    ok = mgq.attention_ring(q, ring, ring, 1000, window=127)   # reach 128 fits
    torch.cuda.synchronize()
    assert torch.all(ok == 0)


def test_decode_steps_on_a_ring_match_oracle():
    """A decode loop on a ring of 192 slots with a window of 150: each step
    appends 1-3 tokens at position p (slot (p + l) % 192) and attends; the
    oracle keeps the whole sequence in order."""
    b, hq, hkv, d, slots, window = 2, 8, 2, 128, 192, 150
    g = torch.Generator().manual_seed(7)
    seq_k = torch.randn(b, 400, hkv, d, generator=g).bfloat16()   # keys in order, page layout
    seq_v = torch.randn(b, 400, hkv, d, generator=g).bfloat16()
    pos = 300
    # the ring after the first 300 tokens: slot j % 192 holds key j
    ring_k = torch.zeros(b, slots, hkv, d, dtype=torch.bfloat16)
    ring_v = torch.zeros_like(ring_k)
    for j in range(pos - slots, pos):
        ring_k[:, j % slots] = seq_k[:, j]
        ring_v[:, j % slots] = seq_v[:, j]
    rk, rv = ring_k.cuda(), ring_v.cuda()
    for step, length in enumerate([1, 3, 2, 1, 3]):
        qs = torch.randn(b, hq, length, d, generator=g).bfloat16()
        new_k = seq_k[:, pos:pos + length].float()       # fp32 tokens, as on the KV-cache page
        new_v = seq_v[:, pos:pos + length].float()
        out = mgq.decode_append(qs.cuda(), rk, rv, new_k.cuda(), new_v.cuda(), pos,
                                seq_major=True, ring=True, causal=True, window=window)
        torch.cuda.synchronize()
        pos += length
        k_lin = seq_k[:, :pos].transpose(1, 2).contiguous()
        v_lin = seq_v[:, :pos].transpose(1, 2).contiguous()
        want = oracle.attention(qs, k_lin, v_lin, causal=True, window=window, softcap=None)
        assert_close(out, want, f"ring decode step {step}")
        # the ring now holds the last 192 keys: slot j % 192 == key j
        host = rk.cpu()
        for j in range(pos - slots, pos):
            assert torch.equal(host[:, j % slots], seq_k[:, j])
