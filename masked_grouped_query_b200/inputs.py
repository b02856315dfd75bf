"""Seeded synthetic inputs and the named workloads.

This module holds no attention arithmetic: it only draws random numbers and
names shapes.  Both the CUDA path and the fp64 oracle are fed from here.

Recipe: a CPU ``torch.Generator`` seeded with the workload's seed draws
standard-normal fp32 values in the order q, k, v, each rounded to bf16.  The
shapes are the decode / prefill / encoder family of "TPU v6e Masked GQA
Kernel Optimization" ("What You Have": GQA 1:1 to 16:1, optional causal
mask, sliding window and logit softcap, bf16 inputs); the encoder shape is
the SigLIP attention of "Independent attention product layouts" ("SigLIP
batch-1 hardware results": 16 heads, 729 tokens, 72 per head), here at
batch 32.  They stand in for that page's visible/held-out case files, which
are not available.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import torch


@dataclass(frozen=True)
class Workload:
    """One attention problem: the cfg fields of the task's entry point."""

    name: str
    batch: int
    q_len: int
    kv_len: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    causal: bool
    window: int | None
    softcap: float | None
    seed: int

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def cfg(self) -> dict:
        """The cfg dict of the task's ``make_attention(cfg)`` entry point."""
        return dict(batch=self.batch, q_len=self.q_len, kv_len=self.kv_len,
                    num_q_heads=self.num_q_heads,
                    num_kv_heads=self.num_kv_heads, head_dim=self.head_dim,
                    causal=self.causal, window=self.window,
                    softcap=self.softcap, seed=self.seed, name=self.name)


WORKLOADS = {
    "tiny_causal_gqa_prefill": Workload(
        "tiny_causal_gqa_prefill", 1, 128, 128, 4, 1, 128, True, None, None, 0),
    "gqa_decode": Workload(
        "gqa_decode", 16, 1, 8192, 32, 8, 128, True, None, None, 1),
    "long_window_softcap_prefill": Workload(
        "long_window_softcap_prefill", 2, 4096, 4096, 32, 4, 128, True, 1024,
        50.0, 2),
    "siglip_encoder": Workload(
        "siglip_encoder", 32, 729, 729, 16, 16, 72, False, None, None, 3),
    "long_context_decode_16to1": Workload(
        "long_context_decode_16to1", 8, 4, 32768, 64, 4, 128, True, 4096,
        30.0, 4),
}

# Workload order matches the configuration list it mirrors.
WORKLOAD_ORDER = list(WORKLOADS)


def make_inputs(w: Workload, seed: int | None = None, q_scale: float = 1.0):
    """Seeded bf16 CPU tensors (q, k, v) for workload ``w``.

    ``q_scale`` multiplies q before rounding (used to drive the softcap into
    saturation).
    """
    g = torch.Generator().manual_seed(w.seed if seed is None else seed)
    qs = (w.batch, w.num_q_heads, w.q_len, w.head_dim)
    ks = (w.batch, w.num_kv_heads, w.kv_len, w.head_dim)
    q = torch.randn(qs, generator=g, dtype=torch.float32)
    if q_scale != 1.0:
        q = q * q_scale
    q = q.to(torch.bfloat16)
    k = torch.randn(ks, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(ks, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


def make_inputs_device(w: Workload, device, seed: int | None = None):
    """Seeded bf16 inputs drawn directly on ``device`` (benchmark sizes).

    The values differ from ``make_inputs`` (a different generator); parity
    tests that compare against the oracle copy these tensors back.
    """
    g = torch.Generator(device=device).manual_seed(w.seed if seed is None else seed)
    qs = (w.batch, w.num_q_heads, w.q_len, w.head_dim)
    ks = (w.batch, w.num_kv_heads, w.kv_len, w.head_dim)
    q = torch.randn(qs, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn(ks, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(ks, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    return q, k, v


@dataclass(frozen=True)
class CacheStep:
    """One decode step on a KV cache: ``count`` new tokens appended at
    ``position`` into caches of ``slots`` slots, then attended by the same
    tokens' queries over slots [0, position + count)."""

    name: str
    batch: int
    slots: int
    position: int
    count: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    causal: bool
    window: int | None
    softcap: float | None
    seed: int

    @property
    def kv_len(self) -> int:
        return self.position + self.count


# The grouped-query decode shape above, run on a cache in the KV-cache page's
# (batch, slots, heads, head_dim) layout: the 8192th token is appended and
# attends to all 8192 slots.
CACHE_STEPS = {
    "gqa_decode_append": CacheStep(
        "gqa_decode_append", 16, 8192, 8191, 1, 32, 8, 128, True, None, None, 5),
}


# Single-token grouped-query decode over a 4096-key sliding window kept in a
# ring of 4096 slots (key j in slot j % 4096) at absolute position 100000.
RING_STEPS = {
    "gqa_decode_ring_window": dict(batch=16, q_len=1, kv_len=100000, slots=4096, num_q_heads=32,
                                   num_kv_heads=8, head_dim=128, causal=True, window=4096,
                                   softcap=None, seed=6),
}


def make_cache_inputs(batch: int, slots: int, heads: int, head_dim: int, count: int, *,
                      cache_dtype=torch.bfloat16, new_dtype=torch.float32, seed: int = 0,
                      num_q_heads: int | None = None, device="cpu"):
    """Seeded caches and new tokens in the KV-cache page's layouts.

    Returns a dict with k_cache, v_cache (batch, slots, heads, head_dim) in
    ``cache_dtype``; new_k, new_v (batch, count, heads, head_dim) in
    ``new_dtype`` (fp32 on the page); and, when ``num_q_heads`` is given, q
    (batch, num_q_heads, count, head_dim) bf16.  Standard-normal draws in the
    order k_cache, v_cache, new_k, new_v, q.
    """
    gen_dev = "cpu" if str(device) == "cpu" else device
    g = torch.Generator(device=gen_dev).manual_seed(seed)

    def draw(shape, dtype):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        return x if dtype == torch.float32 else x.to(dtype)

    cs = (batch, slots, heads, head_dim)
    ns = (batch, count, heads, head_dim)
    out = dict(k_cache=draw(cs, cache_dtype), v_cache=draw(cs, cache_dtype),
               new_k=draw(ns, new_dtype), new_v=draw(ns, new_dtype))
    if num_q_heads is not None:
        out["q"] = draw((batch, num_q_heads, count, head_dim), torch.bfloat16)
    return out
