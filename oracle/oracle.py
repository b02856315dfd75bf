"""fp64 CPU oracle for masked grouped-query attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never does, and shares no code with it.

Two independent restatements of the same definition live here:

* ``attention_rows`` / ``attention`` -- ctypes front end of ``gqa_oracle.c``
  (fp64, OpenMP over rows; handles the full workload sizes row by row);
* ``attention_numpy`` -- a numpy fp64 twin written per (batch, head) with
  whole-matrix operations, for tiny shapes.

The computation follows "TPU v6e Masked GQA Kernel Optimization" ("What You
Have": the family -- GQA 1:1 to 16:1, optional causal mask, sliding window
and logit softcap; "What You Submit": bf16 in, q's shape out) and the
"Independent attention product layouts" flowchart (QK scores, a softmax over
complete rows, PV, normalise).  The mask alignment, window bounds, head
mapping, scale and empty-row readings are stated in ``gqa_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "gqa_oracle.c")
LIBRARY = os.path.join(_HERE, "libgqa_oracle.so")

F64 = 0
BF16 = 1

_lock = threading.Lock()
_lib = None


def compile_oracle(source: str = SOURCE, output: str = LIBRARY) -> str:
    """Compile an oracle source file into a shared library with gcc/OpenMP."""
    cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99", source,
           "-o", output, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return output


def build() -> str:
    """Build ``libgqa_oracle.so`` next to its source (idempotent)."""
    if (not os.path.exists(LIBRARY)
            or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)):
        compile_oracle()
    return LIBRARY


def load(path: str | None = None) -> ctypes.CDLL:
    """Load an oracle library (the built one by default)."""
    lib = ctypes.CDLL(path or build())
    fn = lib.oracle_gqa_attn_rows
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                   ctypes.c_int] + [ctypes.c_int] * 8 + [
                       ctypes.c_double, ctypes.c_void_p, ctypes.c_int64,
                       ctypes.c_void_p, ctypes.c_int]
    lib.oracle_max_threads.restype = ctypes.c_int
    return lib


def _default_lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            _lib = load()
        return _lib


def _as_buffer(t):
    """Return (contiguous array keeping the memory alive, format code)."""
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy(), BF16
        return t.to(torch.float64).numpy(), F64
    a = np.ascontiguousarray(np.asarray(t, dtype=np.float64))
    return a, F64


def attention_rows(q, k, v, *, causal: bool, window: int | None,
                   softcap: float | None, rows=None, threads: int = 0,
                   lib: ctypes.CDLL | None = None) -> np.ndarray:
    """fp64 output rows of masked GQA attention.

    q: (B, Hq, Lq, D); k, v: (B, Hkv, Lk, D), as torch tensors (bf16 or any
    float dtype) or numpy arrays.  ``rows`` lists flat row ids
    ``(b * Hq + h) * Lq + i``; ``None`` means all rows, returned in q's shape.
    """
    lib = lib or _default_lib()
    qa, fq = _as_buffer(q)
    ka, fk = _as_buffer(k)
    va, fv = _as_buffer(v)
    if not (fq == fk == fv):
        raise TypeError("q, k, v must share one element format")
    batch, hq, lq, d = qa.shape
    bk, hkv, lk, dk = ka.shape
    if va.shape != ka.shape or bk != batch or dk != d:
        raise ValueError("shape mismatch between q, k, v")
    win = 0 if window is None else int(window)
    cap = 0.0 if softcap is None else float(softcap)
    if rows is None:
        out = np.empty((batch, hq, lq, d), dtype=np.float64)
        rptr, n = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.empty((r.size, d), dtype=np.float64)
        rptr, n = r.ctypes.data, r.size
    if out.size == 0:
        return out
    rc = lib.oracle_gqa_attn_rows(
        qa.ctypes.data, ka.ctypes.data if ka.size else None,
        va.ctypes.data if va.size else None, fq, batch, lq, lk, hq, hkv, d,
        int(bool(causal)), win, cap, rptr, n, out.ctypes.data, int(threads))
    if rc != 0:
        raise ValueError(f"oracle rejected the arguments (rc={rc})")
    return out


def attention(q, k, v, *, causal, window, softcap, threads: int = 0,
              lib=None) -> np.ndarray:
    """Full fp64 output with q's shape."""
    return attention_rows(q, k, v, causal=causal, window=window,
                          softcap=softcap, rows=None, threads=threads, lib=lib)


def max_threads() -> int:
    return int(_default_lib().oracle_max_threads())


def attention_numpy(q, k, v, *, causal: bool, window: int | None,
                    softcap: float | None) -> np.ndarray:
    """Numpy fp64 twin of the oracle for tiny shapes (whole-matrix form).

    Per (b, h): logits = q_h k_g^T / sqrt(D) with g = h // (Hq/Hkv); capped
    logits c = s * tanh(logits / s) when a softcap s is given; the visibility
    matrix from the bottom-right aligned causal/window rule; a softmax over
    each row's visible entries; rows with none visible are zero.
    """
    def f64(t):
        if isinstance(t, torch.Tensor):
            return t.detach().cpu().to(torch.float64).numpy()
        return np.asarray(t, dtype=np.float64)

    qn, kn, vn = f64(q), f64(k), f64(v)
    batch, hq, lq, d = qn.shape
    hkv, lk = kn.shape[1], kn.shape[2]
    group = hq // hkv
    qpos = (lk - lq) + np.arange(lq)[:, None]
    j = np.arange(lk)[None, :]
    vis = np.ones((lq, lk), dtype=bool)
    if causal:
        vis &= j <= qpos
    if window is not None and window > 0:
        vis &= (qpos - j >= 0) & (qpos - j < window)
    out = np.zeros((batch, hq, lq, d), dtype=np.float64)
    for b in range(batch):
        for h in range(hq):
            g = h // group
            s = qn[b, h] @ kn[b, g].T / np.sqrt(d)
            if softcap is not None and softcap > 0:
                s = softcap * np.tanh(s / softcap)
            s = np.where(vis, s, -np.inf)
            m = s.max(axis=1, keepdims=True) if lk else np.full((lq, 1), -np.inf)
            has = np.isfinite(m)
            w = np.where(vis, np.exp(s - np.where(has, m, 0.0)), 0.0)
            den = w.sum(axis=1, keepdims=True)
            o = (w @ vn[b, g]) / np.where(has, den, 1.0)
            out[b, h] = np.where(has, o, 0.0)
    return out


if __name__ == "__main__":  # pragma: no cover - manual build helper
    print(build(), file=sys.stderr)
