"""The tcgen05 prefill kernel on small cases first (GPU): one tile, two tiles
per CTA in both pairing modes, a ragged last tile, padded head_dim, masks.
Each case is also run through the split-KV decode kernel; both must meet
the oracle bar."""
import numpy as np
import pytest
import torch

import masked_grouped_query_b200 as mgq
from masked_grouped_query_b200.inputs import Workload, make_inputs
from oracle import oracle

pytestmark = pytest.mark.gpu

CASES = [
    # (batch, q_len, kv_len, hq, hkv, d, causal, window, softcap)
    (1, 128, 128, 1, 1, 128, False, None, None),   # one tile, one K/V tile
    (1, 128, 128, 2, 1, 128, True, None, None),    # head pair, causal
    (1, 256, 256, 2, 2, 64, False, None, None),    # consecutive tiles, D = 64
    (1, 200, 300, 1, 1, 128, True, 50, 30.0),      # ragged tile, window, softcap
    (2, 100, 100, 4, 2, 72, False, None, None),    # tiles straddle heads, D = 72
    (1, 729, 729, 2, 2, 72, False, None, None),    # encoder shape, 89-row last tile
    (1, 384, 1000, 8, 1, 128, True, 256, 50.0),    # 8:1 GQA, window + softcap
    (1, 130, 40, 2, 1, 32, True, None, None),      # q_len > kv_len, small D
    (1, 512, 512, 4, 2, 96, True, 1, None),        # window 1 (diagonal)
]


def _check(w, path):
    q, k, v = make_inputs(w)
    mgq.set_override("force_path", path)
    try:
        out = mgq.attention(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, window=w.window,
                            softcap=w.softcap)
        torch.cuda.synchronize()
    finally:
        mgq.set_override("force_path", 0)
    want = oracle.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap)
    got = out.float().cpu().numpy()
    assert np.isfinite(got).all()
    err = np.abs(got - want)
    bad = err > 2e-2 + 2e-2 * np.abs(want)
    assert not bad.any(), f"path {path}: {bad.sum()} bad of {bad.size}, max err {err.max():.4g}"
    return out


@pytest.mark.parametrize("cfg", CASES, ids=[str(c) for c in CASES])
def test_prefill_kernel_small(cfg):
    b, lq, lk, hq, hkv, d, causal, window, cap = cfg
    w = Workload("pf", b, lq, lk, hq, hkv, d, causal, window, cap, seed=lq + lk + d)
    plan = mgq.describe(b, lq, lk, hq, hkv, d, causal, window, cap)
    _check(w, 2)
    _check(w, 1)
    assert mgq.status() & 0x1f == 0, plan
