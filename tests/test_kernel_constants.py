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
