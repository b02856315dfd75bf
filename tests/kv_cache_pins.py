"""Pins for the KV-cache update oracle: checks against things other than it.

Each pin takes the oracle module (``oracle.kv_cache`` or a planted mutant of
it) and raises AssertionError on a mismatch.  They pin it to:

* closed forms of round-to-nearest-even bf16 (ties, carries into the
  exponent, overflow to infinity, subnormals, signed zero, NaN);
* a library routine: torch's float32 -> bfloat16 conversion on values of
  every magnitude, including exact ties;
* the hand-worked updates of ``golden/kv_update_hand_examples.json``;
* the three worked examples the page prints ("KV Cache Update at a
  Position", "Examples"), in ``golden/kv_update_page_examples.json``;
* invariants of the update ("KV Cache Update at a Position", TensorTonic):
  slots outside [position, position + L) are untouched bit for bit, the new
  block equals the converted new vectors concatenated after the old prefix,
  the returned length is position + L, and bf16 -> fp32 -> bf16 is the
  identity on every non-NaN bf16 pattern;
* for the ring variant: a hand-worked ring (slot j % S holds key j), and a
  replay in which a ring and a plain growing sequence receive the same
  appends in chunks of random sizes -- the ring must read back as the last
  S keys of the sequence after every step.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                      "kv_update_hand_examples.json")
PAGE_EXAMPLES = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                             "kv_update_page_examples.json")


def _f32(x):
    return np.array(x, dtype=np.float32)


def pin_rounding_closed_forms(kc):
    cases = [  # (fp32 value, bf16 bits)
        (1.0, 0x3F80), (1.0 + 2.0 ** -8, 0x3F80), (1.0 + 3 * 2.0 ** -8, 0x3F82),
        (1.0 + 2.0 ** -8 + 2.0 ** -23, 0x3F81), (-2.5, 0xC020), (0.0, 0x0000),
        (-0.0, 0x8000), (float("inf"), 0x7F80), (float("-inf"), 0xFF80),
        (float(np.finfo(np.float32).max), 0x7F80),        # carries past the largest bf16
        ((2.0 - 2.0 ** -7) * 2.0 ** 127, 0x7F7F),         # the largest bf16, exact
        (2.0 ** -133, 0x0001), (2.0 ** -149, 0x0000),     # bf16 subnormal; f32 tiny
        (2.0 ** -126 * (1 - 2.0 ** -8), 0x0080),          # subnormal rounding up to normal
        (65792.0, 0x4780), (65793.0, 0x4781),
    ]
    for x, want in cases:
        got = int(kc.f32_to_bf16_bits(_f32([x]))[0])
        assert got == want, f"bf16({x!r}) = {got:#06x}, expected {want:#06x}"
    n = kc.f32_to_bf16_bits(_f32([float("nan"), -float("nan")]))
    assert np.isnan(kc.bf16_bits_to_f32(n)).all()


def pin_rounding_matches_torch(kc):
    rng = np.random.default_rng(7)
    mags = 2.0 ** rng.integers(-140, 126, size=20000)
    x = (rng.standard_normal(20000) * mags).astype(np.float32)
    # exact ties: a random bf16 value plus half its ulp
    t = rng.integers(0, 0x7F7F, size=5000).astype(np.uint32) << 16
    ties = (t | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -ties])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = kc.f32_to_bf16_bits(x)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first at {x[bad[0]]!r}"


def pin_round_trip_identity(kc):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = kc.bf16_bits_to_f32(bits)
    keep = ~np.isnan(f)
    assert np.array_equal(kc.f32_to_bf16_bits(f[keep]), bits[keep])
    # widening is exact: the float32 bits are the bf16 bits followed by 16 zeros
    assert np.array_equal(f[keep].view(np.uint32) >> 16, bits[keep].astype(np.uint32))


def _as_cache(values, dtype, kc):
    a = _f32(values)
    return kc.f32_to_bf16_bits(a) if dtype == "bf16" else a


def _widen(a, kc):
    return kc.bf16_bits_to_f32(a) if a.dtype == np.uint16 else a


def pin_hand_examples(kc, path=GOLDEN):
    with open(path) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        k0 = _as_cache(c["key_cache"], c["cache_dtype"], kc)
        v0 = _as_cache(c["value_cache"], c["cache_dtype"], kc)
        k1, v1, length = kc.kv_update(k0, v0, _f32(c["new_keys"]), _f32(c["new_values"]),
                                      c["position"])
        assert length == c["expected_length"], c["name"]
        for got, want in ((k1, c["expected_key_cache"]), (v1, c["expected_value_cache"])):
            g, w = _widen(got, kc), _f32(want)
            assert np.array_equal(g, w), f"{c['name']}: {g.tolist()} != {w.tolist()}"
            assert np.array_equal(np.signbit(g), np.signbit(w)), f"{c['name']}: zero signs"
        assert k1.dtype == k0.dtype and k1.shape == k0.shape


def pin_page_examples(kc):
    """The page's printed inputs give the page's printed outputs."""
    pin_hand_examples(kc, PAGE_EXAMPLES)


def pin_update_invariants(kc):
    rng = np.random.default_rng(3)
    for cache_dtype in ("f32", "bf16"):
        for (b, s, h, d, length, pos) in [(2, 9, 3, 4, 2, 5), (1, 4, 1, 8, 4, 0),
                                          (3, 6, 2, 2, 1, 5), (2, 5, 2, 4, 0, 3)]:
            k0 = rng.standard_normal((b, s, h, d)).astype(np.float32)
            v0 = rng.standard_normal((b, s, h, d)).astype(np.float32)
            if cache_dtype == "bf16":
                k0, v0 = kc.f32_to_bf16_bits(k0), kc.f32_to_bf16_bits(v0)
            nk = rng.standard_normal((b, length, h, d)).astype(np.float32)
            nv = rng.standard_normal((b, length, h, d)).astype(np.float32)
            k1, v1, n = kc.kv_update(k0, v0, nk, nv, pos)
            assert n == pos + length
            for old, new, tok in ((k0, k1, nk), (v0, v1, nv)):
                conv = (torch.from_numpy(tok).to(torch.bfloat16).view(torch.int16).numpy()
                        .view(np.uint16) if cache_dtype == "bf16" else tok)
                assert np.array_equal(new[:, :pos], old[:, :pos])
                assert np.array_equal(new[:, pos + length:], old[:, pos + length:])
                assert np.array_equal(new[:, :pos + length],
                                      np.concatenate([old[:, :pos], conv], axis=1))
            assert not np.shares_memory(k1, k0)


def pin_ring_hand_example(kc):
    # S = 4 slots, keys 0..5 appended one at a time with value = key index:
    # slot j % 4 holds key j, so slots 0..3 hold 4, 5, 2, 3 and the stored
    # keys in order are 2, 3, 4, 5.
    ring = np.zeros((1, 4, 1, 1), np.float32)
    for j in range(6):
        tok = np.full((1, 1, 1, 1), float(j), np.float32)
        ring, _, n = kc.ring_update(ring, ring, tok, tok, j)
        assert n == j + 1
    assert ring[0, :, 0, 0].tolist() == [4.0, 5.0, 2.0, 3.0]
    seq = kc.ring_sequence(ring, 6, fill=-1.0)
    assert seq[0, :, 0, 0].tolist() == [-1.0, -1.0, 2.0, 3.0, 4.0, 5.0]


def pin_ring_replays_sequence(kc):
    rng = np.random.default_rng(11)
    for s_slots in (4, 8):
        b, h, d = 2, 3, 4
        ring = np.zeros((b, s_slots, h, d), np.float32)
        vring = np.zeros_like(ring)
        seq = np.zeros((b, 0, h, d), np.float32)
        n = 0
        while n < 30:
            length = int(rng.integers(1, s_slots + 1))
            nk = rng.standard_normal((b, length, h, d)).astype(np.float32)
            ring, vring, n2 = kc.ring_update(ring, vring, nk, -nk, n)
            assert n2 == n + length
            n = n2
            seq = np.concatenate([seq, nk], axis=1)
            keep = min(n, s_slots)
            got = kc.ring_sequence(ring, n)
            assert np.array_equal(got[:, n - keep:], seq[:, n - keep:]), (s_slots, n)
            assert np.array_equal(kc.ring_sequence(vring, n)[:, n - keep:], -seq[:, n - keep:])


ALL_PINS = [pin_rounding_closed_forms, pin_rounding_matches_torch, pin_round_trip_identity,
            pin_hand_examples, pin_page_examples, pin_update_invariants, pin_ring_hand_example,
            pin_ring_replays_sequence]
