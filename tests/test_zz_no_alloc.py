"""gqa_attn_fwd_static_scratch: the entry point that allocates no device memory.

Some callers cannot call cudaMalloc -- their device memory is all handed to
their own pool, or they cannot take the synchronisation an allocation may
cause -- so this variant of the split-KV decode path keeps its split
partials and tickets in one fixed device array inside the library instead of
a workspace allocated on first need.  These tests call it through the C ABI,
twice in a row (the array keeps the previous call's contents), and compare
each result with gqa_attn_fwd's and with the fp64 oracle, within the parity
tolerance (rtol = atol = 2e-2).  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from masked_grouped_query_b200 import _lib
from masked_grouped_query_b200.inputs import Workload, make_inputs
from oracle import oracle

pytestmark = pytest.mark.gpu

P = ctypes.c_void_p


def _call(fn, w, q, k, v, out):
    return fn(P(q.data_ptr()), P(k.data_ptr()), P(v.data_ptr()), P(out.data_ptr()),
              w.batch, w.q_len, w.kv_len, w.num_q_heads, w.num_kv_heads, w.head_dim,
              int(w.causal), int(w.window or 0), float(w.softcap or 0.0),
              P(torch.cuda.current_stream().cuda_stream))


CASES = [
    # decode, 4:1 GQA, 32 (batch, kv head) units: five key splits each
    Workload("c2like", 4, 1, 8192, 32, 8, 128, True, None, None, 41),
    # multi-token 16:1 decode with window and softcap (partials ~4.5 MB)
    Workload("c5like", 2, 4, 8192, 64, 4, 128, True, 4096, 30.0, 42),
    # one split: no scratch used at all
    Workload("single", 1, 2, 100, 8, 2, 64, True, None, None, 43),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_static_scratch_matches_gqa_attn_fwd_twice(w):
    lib = _lib.load()
    qh, kh, vh = make_inputs(w)
    exact = oracle.attention(qh, kh, vh, causal=w.causal, window=w.window, softcap=w.softcap)
    q, k, v = qh.cuda(), kh.cuda(), vh.cuda()
    ref = torch.empty_like(q)
    assert _call(lib.gqa_attn_fwd, w, q, k, v, ref) == 0
    torch.cuda.synchronize()
    want = ref.float().cpu().numpy()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        rc = _call(lib.gqa_attn_fwd_static_scratch, w, q, k, v, out)
        assert rc == 0, lib.gqa_attn_last_error_detail().decode()
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all()
        np.testing.assert_allclose(got, want, rtol=2e-2, atol=2e-2)
        # and against the oracle: elementwise |got - exact| <= 2e-2 + 2e-2 |exact|
        np.testing.assert_allclose(got, exact, rtol=2e-2, atol=2e-2)
    assert lib.gqa_attn_status() & 0x1f == 0


def test_static_scratch_rejects_plans_beyond_its_size():
    lib = _lib.load()
    # One key tile per split (the tuning override) at head_dim 256 and 64 rows
    # per kv head: 2 kv heads x 128 splits x 64 rows x 256 fp32 = 16.8 MB > 8 MiB.
    w = Workload("big", 1, 4, 8192, 32, 2, 256, True, None, None, 44)
    q = torch.zeros(w.batch, w.num_q_heads, w.q_len, w.head_dim, dtype=torch.bfloat16,
                    device="cuda")
    k = torch.zeros(w.batch, w.num_kv_heads, w.kv_len, w.head_dim, dtype=torch.bfloat16,
                    device="cuda")
    out = torch.empty_like(q)
    assert lib.gqa_attn_set_override(2, 1) == 0
    try:
        rc = _call(lib.gqa_attn_fwd_static_scratch, w, q, k, k, out)
    finally:
        lib.gqa_attn_set_override(2, 0)
    assert rc == -10
    assert "static scratch too small" in lib.gqa_attn_last_error_detail().decode()
