"""KV-cache update oracle (numpy) -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module; the CUDA library and its binding never
do, and share no code with it.

Follows "KV Cache Update at a Position" (TensorTonic; problem statement,
returned values and constraints): key and value caches of shape (B, S, H, D)
receive the keys and values of L new tokens, (B, L, H, D), at slots
position .. position + L - 1 of every batch row and head, in order; each new
vector is first converted to the cache dtype; every other slot keeps its old
contents; the returned length is position + L.

Representation: an fp32 cache is a float32 array; a bf16 cache is a uint16
array of bf16 bit patterns (numpy has no bf16 type).  New vectors are
float32 (the page's), or uint16 bf16 patterns.

Readings where the page is silent:
* fp32 -> bf16 conversion rounds to nearest, ties to even (the IEEE default
  the page's astype uses); NaN stays NaN (its payload is not fixed), +-inf
  stay infinite, and finite values past bf16's range round to infinity.
* bf16 -> fp32 is exact (the page only sends fp32 new vectors; bf16 new
  vectors are this library's addition).
"""
from __future__ import annotations

import numpy as np

BF16 = "bf16"
F32 = "f32"


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, nearest-even; returns uint16 bit patterns.

    The bf16 value keeps the float32's sign, exponent and top 7 mantissa
    bits; the 16 dropped bits decide the rounding: above half an ulp rounds
    up, below rounds down, exactly half rounds to the even neighbour.  A
    carry out of the mantissa moves into the exponent, which is how the
    largest values become infinity.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    upper = bits >> 16
    lower = bits & 0xFFFF
    half = 0x8000
    round_up = (lower > half) | ((lower == half) & ((upper & 1) == 1))
    out = (upper + round_up.astype(np.uint64)) & 0xFFFF
    nan = np.isnan(x)
    out[nan] = (upper[nan] | 0x0040) & 0xFFFF  # keep the sign, force a quiet NaN
    return out.astype(np.uint16).reshape(x.shape)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).reshape(b.shape)


def convert(new: np.ndarray, cache_dtype: str) -> np.ndarray:
    """The page's conversion of the new vectors to the cache dtype."""
    if cache_dtype == BF16:
        return new.copy() if new.dtype == np.uint16 else f32_to_bf16_bits(new)
    if cache_dtype == F32:
        return bf16_bits_to_f32(new) if new.dtype == np.uint16 else new.astype(np.float32)
    raise ValueError(cache_dtype)


def kv_update(key_cache: np.ndarray, value_cache: np.ndarray, new_keys: np.ndarray,
              new_values: np.ndarray, position: int):
    """Return (key_cache', value_cache', length) for caches (B, S, H, D) and
    new vectors (B, L, H, D); the inputs are not modified."""
    cache_dtype = BF16 if key_cache.dtype == np.uint16 else F32
    b, s, h, d = key_cache.shape
    nb, length, nh, nd = new_keys.shape
    if (nb, nh, nd) != (b, h, d) or value_cache.shape != key_cache.shape:
        raise ValueError("shape mismatch")
    if not 0 <= position <= s - length:
        raise ValueError("the new block must fit inside the cache")
    kc = key_cache.copy()
    vc = value_cache.copy()
    kc[:, position:position + length] = convert(new_keys, cache_dtype)
    vc[:, position:position + length] = convert(new_values, cache_dtype)
    return kc, vc, position + length


def ring_update(key_ring: np.ndarray, value_ring: np.ndarray, new_keys: np.ndarray,
                new_values: np.ndarray, position: int):
    """The update above on ring buffers of S slots: token position + l goes
    to slot (position + l) % S (a circular window, as in "CSA2 attention on
    Metal", TensorFold pull request 1709, "What this changes").  L <= S."""
    cache_dtype = BF16 if key_ring.dtype == np.uint16 else F32
    b, s, h, d = key_ring.shape
    nb, length, nh, nd = new_keys.shape
    if (nb, nh, nd) != (b, h, d) or value_ring.shape != key_ring.shape:
        raise ValueError("shape mismatch")
    if position < 0 or length > s:
        raise ValueError("a block longer than the ring would overwrite itself")
    kc = key_ring.copy()
    vc = value_ring.copy()
    nk = convert(new_keys, cache_dtype)
    nv = convert(new_values, cache_dtype)
    for i in range(length):
        slot = (position + i) % s
        kc[:, slot] = nk[:, i]
        vc[:, slot] = nv[:, i]
    return kc, vc, position + length


def ring_sequence(ring: np.ndarray, kv_len: int, fill=0):
    """Keys (or values) in order from a (B, S, H, D) ring: element j < kv_len
    of the result, (B, kv_len, H, D), is ring slot j % S for the S most recent
    keys j >= kv_len - S; older keys are no longer stored and read as `fill`."""
    b, s, h, d = ring.shape
    out = np.full((b, kv_len, h, d), fill, dtype=ring.dtype)
    for j in range(max(0, kv_len - s), kv_len):
        out[:, j] = ring[:, j % s]
    return out
