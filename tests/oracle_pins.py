"""Pins for the fp64 oracle: checks against things other than the oracle.

Each pin takes ``attn(q, k, v, causal=, window=, softcap=) -> np.ndarray``
(fp64, q's shape) and raises AssertionError on a mismatch.  They pin the
oracle to:

* a library routine in a special case (torch's fp64
  ``scaled_dot_product_attention`` with an explicit boolean mask built from
  ``tril``/``triu`` and repeat-interleaved kv heads, no softcap);
* closed forms (q = 0 gives the mean of v over the visible set; a window of
  1 gives v at qpos; two keys with known logits give a logistic mix; the
  hand-derived cases of ``golden/mask_closed_forms.json``);
* invariants (constant v returns v -- after the constant-input checks of
  "Independent attention product layouts", "SigLIP batch-1 hardware
  results"; masked keys do not matter; GQA equals MHA with repeated kv heads;
  key permutation without a mask; softcap -> infinity equals no softcap);
* the degenerate cases (rows with no visible key are zero, never NaN).

The mask rule being pinned is the bottom-right alignment stated in the
oracle's header.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

MASKS = [(False, None), (True, None), (True, 3), (False, 2), (True, 1),
         (False, 1), (True, 64)]


def visibility(lq: int, lk: int, causal: bool, window) -> torch.Tensor:
    """Boolean (lq, lk) visibility from triangular library masks.

    ``tril(diagonal=lk-lq)`` keeps j <= i + (lk - lq) = qpos (bottom-right
    causal); ``triu(diagonal=lk-lq-w+1)`` keeps j >= qpos - w + 1.
    """
    ones = torch.ones(lq, lk, dtype=torch.bool)
    m = ones.clone()
    if causal or (window is not None and window > 0):
        m &= torch.tril(ones, diagonal=lk - lq)
    if window is not None and window > 0:
        m &= torch.triu(ones, diagonal=lk - lq - window + 1)
    return m


def _rand(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g, dtype=torch.float64) * scale)


def _case(b, hq, hkv, lq, lk, d, seed):
    q = _rand((b, hq, lq, d), seed)
    k = _rand((b, hkv, lk, d), seed + 1)
    v = _rand((b, hkv, lk, d), seed + 2)
    return q, k, v


SHAPES = [  # (b, hq, hkv, lq, lk, d)
    (1, 1, 1, 1, 1, 4), (1, 2, 1, 3, 5, 4), (2, 4, 2, 4, 4, 8),
    (1, 3, 1, 5, 9, 8), (2, 6, 3, 7, 3, 4), (1, 2, 2, 9, 6, 8),
    (1, 4, 1, 2, 9, 4),
]


def pin_sdpa(attn):
    """No softcap: equals torch fp64 SDPA with the explicit mask (visible rows)."""
    seed = 10
    for (b, hq, hkv, lq, lk, d) in SHAPES:
        for causal, window in MASKS:
            q, k, v = _case(b, hq, hkv, lq, lk, d, seed)
            seed += 3
            got = attn(q, k, v, causal=causal, window=window, softcap=None)
            vis = visibility(lq, lk, causal, window)
            g = hq // hkv
            ref = F.scaled_dot_product_attention(
                q, k.repeat_interleave(g, dim=1), v.repeat_interleave(g, dim=1),
                attn_mask=vis).numpy()
            rows = vis.any(dim=1).numpy()
            np.testing.assert_allclose(got[:, :, rows], ref[:, :, rows],
                                       rtol=1e-11, atol=1e-12)
            assert np.all(got[:, :, ~rows] == 0.0)


def pin_constant_v(attn):
    """v constant along keys returns that constant on rows with a visible key."""
    for (b, hq, hkv, lq, lk, d) in SHAPES:
        for causal, window in MASKS:
            q, k, _ = _case(b, hq, hkv, lq, lk, d, 77)
            c = _rand((b, hkv, 1, d), 78)
            v = c.expand(b, hkv, lk, d).contiguous()
            got = attn(q, k, v, causal=causal, window=window, softcap=30.0)
            rows = visibility(lq, lk, causal, window).any(dim=1).numpy()
            g = hq // hkv
            want = c.repeat_interleave(g, dim=1).expand(b, hq, lq, d).numpy()
            np.testing.assert_allclose(got[:, :, rows], want[:, :, rows],
                                       rtol=1e-13, atol=1e-13)


def pin_zero_q_mean(attn):
    """q = 0: every visible logit is 0, so a row is the mean of visible v."""
    for (b, hq, hkv, lq, lk, d) in SHAPES:
        for causal, window in MASKS:
            _, k, v = _case(b, hq, hkv, lq, lk, d, 91)
            q = torch.zeros(b, hq, lq, d, dtype=torch.float64)
            for cap in (None, 20.0):
                got = attn(q, k, v, causal=causal, window=window, softcap=cap)
                vis = visibility(lq, lk, causal, window).to(torch.float64)
                cnt = vis.sum(dim=1, keepdim=True)
                g = hq // hkv
                vr = v.repeat_interleave(g, dim=1)
                mean = (vis @ vr) / torch.where(cnt > 0, cnt, torch.ones_like(cnt))
                np.testing.assert_allclose(got, mean.numpy(), rtol=1e-12,
                                           atol=1e-13)


def pin_golden_mask_cases(attn):
    """Hand-derived closed forms stored in golden/mask_closed_forms.json."""
    with open(os.path.join(GOLDEN, "mask_closed_forms.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        lq, lk, d = c["q_len"], c["kv_len"], c["head_dim"]
        q = torch.zeros(1, 1, lq, d, dtype=torch.float64)
        k = _rand((1, 1, lk, d), 5)
        v = torch.tensor(c["v"], dtype=torch.float64).reshape(1, 1, lk, d)
        got = attn(q, k, v, causal=c["causal"], window=c["window"] or None,
                   softcap=None)
        np.testing.assert_allclose(got[0, 0], np.array(c["expected"], float),
                                   rtol=0, atol=1e-14, err_msg=c["name"])


def pin_window_one(attn):
    """window = 1: each row returns v at its own position (or zeros)."""
    for (b, hq, hkv, lq, lk, d) in SHAPES:
        q, k, v = _case(b, hq, hkv, lq, lk, d, 123)
        got = attn(q, k, v, causal=False, window=1, softcap=None)
        g = hq // hkv
        for i in range(lq):
            qpos = lk - lq + i
            for h in range(hq):
                want = v[:, h // g, qpos] if 0 <= qpos < lk else torch.zeros(b, d, dtype=torch.float64)
                np.testing.assert_allclose(got[:, h, i], want.numpy(), rtol=0,
                                           atol=1e-14)


def pin_masked_key_invariance(attn):
    """Changing k, v at keys a row cannot see leaves that row unchanged."""
    for (b, hq, hkv, lq, lk, d) in SHAPES[1:5]:
        for causal, window in MASKS[1:5]:
            q, k, v = _case(b, hq, hkv, lq, lk, d, 55)
            base = attn(q, k, v, causal=causal, window=window, softcap=40.0)
            vis = visibility(lq, lk, causal, window)
            for i in range(lq):
                hidden = ~vis[i]
                if not hidden.any():
                    continue
                k2, v2 = k.clone(), v.clone()
                k2[:, :, hidden] = _rand(k2[:, :, hidden].shape, 99 + i, 300.0)
                v2[:, :, hidden] = _rand(v2[:, :, hidden].shape, 199 + i, 1e4)
                got = attn(q, k2, v2, causal=causal, window=window, softcap=40.0)
                np.testing.assert_allclose(got[:, :, i], base[:, :, i],
                                           rtol=1e-13, atol=1e-13)


def pin_gqa_equals_mha(attn):
    """GQA equals MHA over kv heads repeat-interleaved by the group size."""
    for (b, hq, hkv, lq, lk, d) in SHAPES:
        if hq == hkv:
            continue
        q, k, v = _case(b, hq, hkv, lq, lk, d, 31)
        g = hq // hkv
        for causal, window in MASKS[:4]:
            a = attn(q, k, v, causal=causal, window=window, softcap=25.0)
            m = attn(q, k.repeat_interleave(g, dim=1), v.repeat_interleave(g, dim=1),
                     causal=causal, window=window, softcap=25.0)
            np.testing.assert_allclose(a, m, rtol=1e-13, atol=1e-13)


def _two_key_case(d, alpha, beta_a, beta_b, seed):
    q = torch.zeros(1, 1, 1, d, dtype=torch.float64)
    q[..., 0] = alpha
    k = torch.zeros(1, 1, 2, d, dtype=torch.float64)
    k[0, 0, 0, 0] = beta_a
    k[0, 0, 1, 0] = beta_b
    v = _rand((1, 1, 2, d), seed)
    return q, k, v


def pin_softcap_two_keys(attn):
    """Two keys with exact logits: o = sig(c_a - c_b) v_a + sig(c_b - c_a) v_b.

    c = s * tanh(x / s), x = alpha * beta / sqrt(D) with the logical D
    (D = 72 pins the unpadded scale).  Saturating logits (|x| >> s) make a
    dropped or misplaced softcap visible.
    """
    cases = [  # d, alpha, beta_a, beta_b, softcap
        (8, 10.0, 3.0, -2.0, 5.0), (8, 40.0, 30.0, 10.0, 30.0),
        (72, 60.0, 50.0, 20.0, 50.0), (72, 3.0, 2.0, 1.0, None),
        (128, 100.0, 80.0, -80.0, 30.0), (128, 1.5, 0.7, 0.2, 50.0),
        (16, 20.0, 9.0, 8.0, 1.0),
    ]
    for n, (d, al, ba, bb, s) in enumerate(cases):
        q, k, v = _two_key_case(d, al, ba, bb, 400 + n)
        got = attn(q, k, v, causal=False, window=None, softcap=s)
        xa, xb = al * ba / np.sqrt(d), al * bb / np.sqrt(d)
        if s is not None:
            xa, xb = s * np.tanh(xa / s), s * np.tanh(xb / s)
        wa = 1.0 / (1.0 + np.exp(xb - xa))
        want = wa * v[0, 0, 0].numpy() + (1.0 - wa) * v[0, 0, 1].numpy()
        np.testing.assert_allclose(got[0, 0, 0], want, rtol=1e-12, atol=1e-13)


def pin_softcap_limit(attn):
    """A huge softcap reproduces the uncapped result."""
    for (b, hq, hkv, lq, lk, d) in SHAPES[:4]:
        q, k, v = _case(b, hq, hkv, lq, lk, d, 61)
        a = attn(q, k, v, causal=True, window=None, softcap=1e9)
        n = attn(q, k, v, causal=True, window=None, softcap=None)
        np.testing.assert_allclose(a, n, rtol=1e-9, atol=1e-10)


def pin_permutation(attn):
    """Without a mask, permuting keys and values jointly changes nothing."""
    for (b, hq, hkv, lq, lk, d) in SHAPES:
        q, k, v = _case(b, hq, hkv, lq, lk, d, 71)
        perm = torch.randperm(lk, generator=torch.Generator().manual_seed(lk))
        a = attn(q, k, v, causal=False, window=None, softcap=15.0)
        p = attn(q, k[:, :, perm], v[:, :, perm], causal=False, window=None,
                 softcap=15.0)
        np.testing.assert_allclose(a, p, rtol=1e-12, atol=1e-13)


def pin_empty_rows(attn):
    """Rows with no visible key are exactly zero; nothing is NaN."""
    q, k, v = _case(1, 4, 2, 6, 3, 8, 81)
    for causal, window in [(True, None), (True, 2), (False, 1)]:
        got = attn(q, k, v, causal=causal, window=window, softcap=10.0)
        assert np.all(np.isfinite(got))
        assert np.all(got[:, :, :3] == 0.0)  # qpos = -3, -2, -1
    empty_k = torch.zeros(1, 2, 0, 8, dtype=torch.float64)
    got = attn(q, empty_k, empty_k, causal=False, window=None, softcap=None)
    assert got.shape == q.shape and np.all(got == 0.0)


ALL_PINS = [pin_sdpa, pin_constant_v, pin_zero_q_mean, pin_golden_mask_cases,
            pin_window_one, pin_masked_key_invariance, pin_gqa_equals_mha,
            pin_softcap_two_keys, pin_softcap_limit, pin_permutation,
            pin_empty_rows]
