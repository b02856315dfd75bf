"""Host-side checks of constants compiled into the CUDA kernels (CPU only)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PTX = os.path.join(ROOT, "masked_grouped_query_b200", "csrc", "ptx.cuh")


def _body(name):
    src = open(PTX).read()
    body = src[src.index(name):]
    return body[:body.index("}\n")]


def test_small_argument_tanh_polynomial_error():
    # y * P(y^2) used for the softcap when |y| <= 1/2.
    c = [float(v) for v in re.findall(r"(-?\d\.\d+)f", _body("float tanh_poly_small(float y)"))]
    c7, c5, c3, c1 = c[:4]
    y = np.linspace(-0.5, 0.5, 200001)
    y2 = y * y
    t = y * (((c7 * y2 + c5) * y2 + c3) * y2 + c1)
    err = np.abs(t - np.tanh(y)).max()
    assert err < 2e-7
    # times the largest softcap of the workloads (50): logit error < 1e-5
    assert 50 * err < 1e-5
