"""Masked grouped-query attention forward for NVIDIA B200 (sm_100a).

``make_attention(cfg)`` returns ``f(q, k, v)`` over bf16 CUDA tensors; every
step of the computation runs in the CUDA library ``libgqa_attn.so`` behind
the C ABI declared in ``include/gqa_attn.h``.  This package only marshals
arguments.  Importing it does not load the library; the first call does, and
raises if the library is missing (there is no CPU fallback).
"""
from .attention import (attention, attention_host, clear_status, describe,  # noqa: F401
                        make_attention, release_workspace, selftest_bounded_wait, set_override,
                        status)
from .inputs import WORKLOADS, Workload, make_inputs  # noqa: F401
from .kv_cache import attention_ring, decode_append, kv_append  # noqa: F401

__all__ = ["attention", "attention_host", "make_attention", "describe", "set_override",
           "status", "clear_status", "release_workspace", "selftest_bounded_wait", "WORKLOADS",
           "Workload",
           "make_inputs", "kv_append", "decode_append", "attention_ring"]
