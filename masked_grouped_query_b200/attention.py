"""Python entry points over the C ABI (argument marshalling only).

``make_attention(cfg)`` mirrors the entry signature of "TPU v6e Masked GQA
Kernel Optimization" ("What You Submit"): it returns ``f(q, k, v)`` taking
bf16 q (batch, num_q_heads, q_len, head_dim) and k, v (batch, num_kv_heads,
kv_len, head_dim) and returning bf16 o with q's shape.  cfg fields: batch,
q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window (None =
no window), softcap (None = no softcap); ``seed`` and ``name`` are accepted
and ignored -- nothing branches on them ("Hard Constraints").
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib


def _stream_handle(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check_tensor(name, t, ndim=4):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _args(window, softcap, causal):
    w = 0 if window is None else int(window)
    s = 0.0 if softcap is None else float(softcap)
    return int(bool(causal)), w, s


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
              window: int | None = None, softcap: float | None = None,
              out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Masked GQA attention forward on the current CUDA device and stream."""
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t)
        if not t.is_cuda:
            raise ValueError(f"{n} must be a CUDA tensor (use attention_host for host buffers)")
    b, hq, lq, d = q.shape
    bk, hkv, lk, dk = k.shape
    if tuple(v.shape) != tuple(k.shape) or bk != b or dk != d:
        raise ValueError(f"shape mismatch: q {tuple(q.shape)}, k {tuple(k.shape)}, "
                         f"v {tuple(v.shape)}")
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_tensor("out", out)
        if out.shape != q.shape or out.device != q.device:
            raise ValueError("out must match q's shape and device")
    c, w, s = _args(window, softcap, causal)
    lib = _lib.load()
    with torch.cuda.device(q.device):
        rc = lib.gqa_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                              b, lq, lk, hq, hkv, d, c, w, s, _stream_handle(stream))
    _lib.check(rc, "gqa_attn_fwd")
    return out


def attention_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool = False,
                   window: int | None = None, softcap: float | None = None,
                   out: torch.Tensor | None = None, device_buffers=None,
                   stream=None) -> torch.Tensor:
    """Masked GQA attention for host (CPU, preferably pinned) tensors.

    Copies q, k, v to ``device_buffers`` (a dict with q, k, v, o device
    tensors; allocated here when omitted), runs the kernel and copies o back
    into ``out`` (pinned when allocated here), all inside the C call
    ``gqa_attn_fwd_host``; returns ``out`` after the stream has finished.
    """
    for n, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(n, t)
        if t.is_cuda:
            raise ValueError(f"{n} must be a host tensor")
    b, hq, lq, d = q.shape
    _, hkv, lk, _ = k.shape
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    if device_buffers is None:
        dev = torch.device("cuda", torch.cuda.current_device())
        device_buffers = {n: torch.empty(t.shape, dtype=t.dtype, device=dev)
                          for n, t in (("q", q), ("k", k), ("v", v), ("o", q))}
    db = device_buffers
    c, w, s = _args(window, softcap, causal)
    lib = _lib.load()
    with torch.cuda.device(db["q"].device):
        rc = lib.gqa_attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   db["q"].data_ptr(), db["k"].data_ptr(), db["v"].data_ptr(),
                                   db["o"].data_ptr(), b, lq, lk, hq, hkv, d, c, w, s,
                                   _stream_handle(stream))
    _lib.check(rc, "gqa_attn_fwd_host")
    return out


def make_attention(cfg: dict):
    """Return ``f(q, k, v) -> o`` for one configuration (bf16 in, bf16 out)."""
    causal = bool(cfg.get("causal", False))
    window = cfg.get("window")
    softcap = cfg.get("softcap")
    expect_q = (cfg["batch"], cfg["num_q_heads"], cfg["q_len"], cfg["head_dim"])
    expect_kv = (cfg["batch"], cfg["num_kv_heads"], cfg["kv_len"], cfg["head_dim"])

    def f(q, k, v):
        if tuple(q.shape) != expect_q or tuple(k.shape) != expect_kv:
            raise ValueError(f"inputs do not match cfg: q {tuple(q.shape)} vs {expect_q}, "
                             f"k {tuple(k.shape)} vs {expect_kv}")
        return attention(q, k, v, causal=causal, window=window, softcap=softcap)

    return f


def describe(batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal=False,
             window=None, softcap=None) -> dict:
    """The launch plan for these sizes on the current device (no launch)."""
    c, w, s = _args(window, softcap, causal)
    outs = [ctypes.c_int(0) for _ in range(4)]
    rc = _lib.load().gqa_attn_describe(batch, q_len, kv_len, num_q_heads, num_kv_heads,
                                       head_dim, c, w, s, *[ctypes.byref(o) for o in outs])
    _lib.check(rc, "gqa_attn_describe")
    path = {0: "none", 1: "decode", 2: "prefill", 3: "zero"}[outs[0].value]
    cluster = ctypes.c_int(0)
    rc = _lib.load().gqa_attn_describe_merge(batch, q_len, kv_len, num_q_heads, num_kv_heads,
                                             head_dim, c, w, s, ctypes.byref(cluster))
    _lib.check(rc, "gqa_attn_describe_merge")
    return dict(path=path, splits=outs[1].value, ctas=outs[2].value, tiles=outs[3].value,
                cluster=cluster.value)


def set_override(key: str, value: int) -> None:
    """Test/tuning knob: ``force_path`` (0 auto, 1 decode, 2 prefill),
    ``tiles_per_split`` (decode, 0 = automatic), ``prefill_splits``
    (tcgen05 kernel, units with one row tile; 0 = automatic) or
    ``prefill_cluster`` (how those splits merge: 0 automatic, -1 always by
    the last CTA of a unit instead of a thread-block cluster) or
    ``softcap_two_pass`` (1: the tcgen05 softcap path takes the row max
    first instead of its fixed exponent base)."""
    k = {"force_path": 1, "tiles_per_split": 2, "prefill_splits": 3, "prefill_cluster": 4,
         "softcap_two_pass": 5}[key]
    _lib.check(_lib.load().gqa_attn_set_override(k, int(value)), "gqa_attn_set_override")


def status() -> int:
    """Sticky device status word (0 = no bounded wait gave up)."""
    return int(_lib.load().gqa_attn_status())


def clear_status() -> None:
    """Reset the status word and the split-ticket counters (after a sync)."""
    _lib.check(_lib.load().gqa_attn_clear_status(), "gqa_attn_clear_status")


def release_workspace() -> None:
    """Free every split workspace the library holds (synchronises)."""
    _lib.check(_lib.load().gqa_attn_release_workspace(), "gqa_attn_release_workspace")


def selftest_bounded_wait(limit_us: int = 1000, stream=None) -> None:
    """Launch the bounded-wait self test (a wait that must give up)."""
    _lib.check(_lib.load().gqa_attn_selftest_bounded_wait(int(limit_us), _stream_handle(stream)),
               "gqa_attn_selftest_bounded_wait")
