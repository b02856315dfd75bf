"""Seeded random shapes through every path against the fp64 oracle (GPU).

Each case draws a batch, GQA group, q and kv lengths, head_dim, mask and
softcap, so the plan lands on the split-KV decode kernel (with or without
splits), the tcgen05 kernel (unsplit, key splits, paired splits, clusters),
the fixed-base and row-max softcap paths, and the deep and shallow decode
rings.  The bar is the attention tolerance of test_parity.
"""
import random

import pytest

from masked_grouped_query_b200.inputs import Workload

from .test_parity import check_workload

pytestmark = pytest.mark.gpu


def _cases(n=80, seed=20261203):
    rng = random.Random(seed)
    out = []
    for i in range(n):
        hkv = rng.choice([1, 2, 4])
        group = rng.choice([1, 2, 4, 8, 16])
        q_len = rng.choice([1, 2, 4, 7, 33, 128, 129, 200, 300])
        kv_len = q_len + rng.choice([0, 1, 63, 64, 200, 511, 900])
        d = rng.choice([64, 72, 80, 96, 128, 128, 256])
        causal = rng.random() < 0.7
        window = rng.choice([None, None, 1, 17, 128, 300])
        softcap = rng.choice([None, None, 5.0, 30.0, 50.0, 70.0, 300.0])
        q_scale = rng.choice([1.0, 1.0, 8.0])
        batch = rng.choice([1, 2, 3])
        out.append((Workload(f"r{i}", batch, q_len, kv_len, group * hkv, hkv, d, causal, window,
                             softcap, 1000 + i), q_scale))
    return out


CASES = _cases()


@pytest.mark.parametrize("case", CASES, ids=[c[0].name for c in CASES])
def test_random_shape_matches_oracle(case):
    w, q_scale = case
    check_workload(w, q_scale=q_scale)
