"""ctypes binding of ``libgqa_attn.so`` (argument marshalling only).

Every function here calls straight into the C ABI of ``include/gqa_attn.h``;
no step of the attention runs in Python.  There is no fallback: when the
library is missing or fails to load, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(PKG, "libgqa_attn.so")

# Symbols exported by the library (the declarations of include/gqa_attn.h).
EXPORTS = (
    "gqa_attn_fwd", "gqa_attn_fwd_host", "gqa_attn_describe",
    "gqa_attn_set_override", "gqa_attn_error_string", "gqa_attn_status",
    "gqa_attn_clear_status", "gqa_attn_selftest_bounded_wait",
    "gqa_attn_version", "gqa_attn_last_error_detail", "gqa_attn_fwd_static_scratch",
    "gqa_attn_kv_append", "gqa_attn_decode_append", "gqa_attn_fwd_ring",
    "gqa_attn_describe_merge", "gqa_attn_release_workspace",
)

_I = ctypes.c_int
_P = ctypes.c_void_p
_F = ctypes.c_float
# batch, q_len, kv_len, num_q_heads, num_kv_heads, head_dim, causal, window, softcap
_DIMS = [_I, _I, _I, _I, _I, _I, _I, _I, _F]

_lock = threading.Lock()
_lib = None


class GqaAttnError(RuntimeError):
    """A non-zero return code of the C library."""

    def __init__(self, code: int, what: str):
        detail = load().gqa_attn_last_error_detail().decode()
        super().__init__(f"{what} failed: {error_string(code)} (code {code})"
                         + (f" [{detail}]" if detail else ""))
        self.code = code


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library once; raise if it is missing (no fallback path)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIBRARY
        if not os.path.exists(p):
            raise RuntimeError(
                f"CUDA library {p} is missing: build it with "
                "`python -m masked_grouped_query_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(p)
        lib.gqa_attn_fwd.restype = _I
        lib.gqa_attn_fwd.argtypes = [_P, _P, _P, _P] + _DIMS + [_P]
        lib.gqa_attn_fwd_host.restype = _I
        lib.gqa_attn_fwd_host.argtypes = [_P] * 8 + _DIMS + [_P]
        lib.gqa_attn_describe.restype = _I
        lib.gqa_attn_describe.argtypes = _DIMS + [ctypes.POINTER(_I)] * 4
        lib.gqa_attn_describe_merge.restype = _I
        lib.gqa_attn_describe_merge.argtypes = _DIMS + [ctypes.POINTER(_I)]
        lib.gqa_attn_release_workspace.restype = _I
        lib.gqa_attn_release_workspace.argtypes = []
        lib.gqa_attn_set_override.restype = _I
        lib.gqa_attn_set_override.argtypes = [_I, _I]
        lib.gqa_attn_error_string.restype = ctypes.c_char_p
        lib.gqa_attn_error_string.argtypes = [_I]
        lib.gqa_attn_status.restype = _I
        lib.gqa_attn_status.argtypes = []
        lib.gqa_attn_clear_status.restype = _I
        lib.gqa_attn_clear_status.argtypes = []
        lib.gqa_attn_selftest_bounded_wait.restype = _I
        lib.gqa_attn_selftest_bounded_wait.argtypes = [_I, _P]
        lib.gqa_attn_version.restype = _I
        lib.gqa_attn_version.argtypes = []
        lib.gqa_attn_last_error_detail.restype = ctypes.c_char_p
        lib.gqa_attn_last_error_detail.argtypes = []
        lib.gqa_attn_fwd_static_scratch.restype = _I
        lib.gqa_attn_fwd_static_scratch.argtypes = [_P, _P, _P, _P] + _DIMS + [_P]
        lib.gqa_attn_kv_append.restype = _I
        lib.gqa_attn_kv_append.argtypes = ([_P] * 4 + [_I] * 6 +
                                           [ctypes.c_uint, ctypes.POINTER(_I), _P])
        lib.gqa_attn_decode_append.restype = _I
        lib.gqa_attn_decode_append.argtypes = ([_P] * 6 + [_I] * 7 +
                                               [ctypes.c_uint, _I, _I, _F, _P])
        lib.gqa_attn_fwd_ring.restype = _I
        lib.gqa_attn_fwd_ring.argtypes = ([_P] * 4 + [_I] * 7 + [ctypes.c_uint, _I, _I, _F, _P])
        if path is None:
            _lib = lib
        return lib


def error_string(code: int) -> str:
    return load().gqa_attn_error_string(int(code)).decode()


def check(code: int, what: str) -> None:
    if code != 0:
        raise GqaAttnError(code, what)
