"""Host-side checks of constants compiled into the CUDA kernels (CPU only)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "masked_grouped_query_b200", "csrc", "ptx.cuh")


def test_small_argument_tanh_polynomial_error():
    # y * P(y^2) used for the softcap when |y| <= 1/2.
    src = open(PTX).read()
    c = {k: float(v) for k, v in re.findall(r"kTanh(C\d) = (-?\d\.\d+)f", src)}
    y = np.linspace(-0.5, 0.5, 200001)
    y2 = y * y
    t = y * (((c["C7"] * y2 + c["C5"]) * y2 + c["C3"]) * y2 + c["C1"])
    err = np.abs(t - np.tanh(y)).max()
    assert err < 2e-7
    # times the largest softcap of the workloads (50): logit error < 1e-5
    assert 50 * err < 1e-5


def test_degree5_tanh_polynomial_error_and_cap_limit():
    # The degree-5 polynomial the kernel uses for softcaps up to kTanh5MaxCap:
    # its error times cap * log2(e) must stay below 2e-3 log2 units there.
    src = open(PTX).read()
    c = {k: float(v) for k, v in re.findall(r"kTanh5(C\d) = (-?\d\.\d+)f", src)}
    cap = float(re.search(r"kTanh5MaxCap = (\d+\.\d+)f", src).group(1))
    y = np.linspace(-0.5, 0.5, 200001)
    y2 = y * y
    t = y * ((c["C5"] * y2 + c["C3"]) * y2 + c["C1"])
    err = np.abs(t - np.tanh(y)).max()
    assert err < 6e-6
    assert cap * np.log2(np.e) * err < 2e-3


def _exp2_consts():
    src = open(PTX).read()
    return {k: float(v) for k, v in re.findall(r"kExp2(C\d) = (-?\d\.\d+(?:e-?\d+)?)f", src)}


def test_exp2_cubic_relative_error():
    # 2^f on [0, 1] from the cubic the softmax uses on the FMA pipe.
    c = _exp2_consts()
    f = np.linspace(0.0, 1.0, 200001)
    p = ((c["C3"] * f + c["C2"]) * f + c["C1"]) * f + c["C0"]
    assert np.abs(p / np.exp2(f) - 1.0).max() < 8e-5


def test_exp2_cody_waite_reconstruction_in_float32():
    # The kernel's steps, in float32 arithmetic: clamp at -126, t = y + 1.5 * 2^23
    # rounded toward -inf (floor(y) in the low mantissa bits), f = y - (t - magic),
    # cubic, then floor(y) << 23 added to the result's bits.
    c = {k: np.float32(v) for k, v in _exp2_consts().items()}
    rng = np.random.default_rng(5)
    y = np.concatenate([rng.uniform(-125.0, 8.0, 400000), np.arange(-125, 9, dtype=np.float64),
                        np.array([-0.0, 1e-7, -1e-7, 7.999999]),
                        rng.uniform(-1e30, -125.0, 1000), np.array([-np.inf])]).astype(np.float32)
    yc = np.maximum(y, np.float32(-126.0))
    magic = np.float32(12582912.0)
    # round toward -inf of y + magic: the exact sum is representable in float64
    exact = yc.astype(np.float64) + 12582912.0
    t = np.floor(exact).astype(np.float32)
    fr = (yc - (t - magic)).astype(np.float32)
    assert ((fr >= 0) & (fr < 1)).all()
    q = ((c["C3"] * fr + c["C2"]) * fr + c["C1"]) * fr + c["C0"]
    bits = q.astype(np.float32).view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    got = bits.view(np.float32).astype(np.float64)
    want = np.exp2(y.astype(np.float64))
    ok = y >= -125
    assert np.abs(got[ok] / want[ok] - 1.0).max() < 8e-5
    # below: finite, non-negative and negligible (under 2^-124)
    assert (got[~ok] >= 0).all() and (got[~ok] < 2.0 ** -124).all()
