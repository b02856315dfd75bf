"""The fp64 oracle against its pins (CPU only).

Both restatements of the definition (the C oracle and its numpy twin) must
pass every pin.  Planted controls: each mutant of the C oracle source --
a plausible mistake compiled into a throw-away library -- must fail at
least one pin, which shows the pins can see that kind of mistake (the
"kernel contract" controls that must go red, "CSA2 attention on Metal",
section "Receipt").
"""
import os

import numpy as np
import pytest
import torch

from oracle import oracle
from tests import oracle_pins as pins


def c_oracle(lib=None):
    def attn(q, k, v, *, causal, window, softcap):
        return oracle.attention(q, k, v, causal=causal, window=window,
                                softcap=softcap, lib=lib)
    return attn


def numpy_oracle(q, k, v, *, causal, window, softcap):
    return oracle.attention_numpy(q, k, v, causal=causal, window=window,
                                  softcap=softcap)


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_c_oracle_pins(pin):
    pin(c_oracle())


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda p: p.__name__)
def test_numpy_oracle_pins(pin):
    pin(numpy_oracle)


def test_c_and_numpy_agree_on_bf16_inputs():
    from masked_grouped_query_b200.inputs import Workload, make_inputs
    for n, (lq, lk, hq, hkv, d, causal, window, cap) in enumerate([
            (5, 9, 4, 1, 16, True, None, None), (9, 9, 6, 2, 8, True, 4, 30.0),
            (1, 33, 8, 2, 24, True, None, 50.0), (7, 7, 2, 2, 72, False, None, None),
            (12, 5, 4, 4, 8, True, 3, 2.0)]):
        w = Workload("t", 2, lq, lk, hq, hkv, d, causal, window, cap, 100 + n)
        q, k, v = make_inputs(w)
        a = oracle.attention(q, k, v, causal=causal, window=window, softcap=cap)
        b = oracle.attention_numpy(q, k, v, causal=causal, window=window,
                                   softcap=cap)
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_row_sampling_matches_full():
    from masked_grouped_query_b200.inputs import Workload, make_inputs
    w = Workload("t", 2, 11, 20, 6, 2, 16, True, 7, 20.0, 9)
    q, k, v = make_inputs(w)
    full = oracle.attention(q, k, v, causal=True, window=7, softcap=20.0)
    rows = np.array([0, 5, 17, 40, 131, 2 * 6 * 11 - 1])
    part = oracle.attention_rows(q, k, v, causal=True, window=7, softcap=20.0,
                                 rows=rows)
    np.testing.assert_array_equal(part, full.reshape(-1, 16)[rows])


def test_oracle_rejects_bad_arguments():
    q = torch.zeros(1, 3, 2, 8, dtype=torch.float64)
    k = torch.zeros(1, 2, 2, 8, dtype=torch.float64)
    with pytest.raises(ValueError):  # 3 q heads over 2 kv heads
        oracle.attention(q, k, k, causal=False, window=None, softcap=None)
    with pytest.raises(ValueError):
        oracle.attention(q[:, :2], k, k, causal=False, window=None, softcap=-1.0)


# (name, text in gqa_oracle.c, replacement) -- plausible mistakes.
MUTANTS = [
    ("top_left_alignment", "long qpos = (long)kv_len - q_len + i;",
     "long qpos = i;"),
    ("window_off_by_one", "(qpos - j) < window", "(qpos - j) <= window"),
    ("kv_head_modulo", "int hk = h / group;", "int hk = h % num_kv_heads;"),
    ("scale_with_padded_dim", "double scale = 1.0 / sqrt((double)head_dim);",
     "double scale = 1.0 / sqrt((double)((head_dim + 15) / 16 * 16));"),
    ("softcap_dropped", "if (softcap > 0.0) s = softcap * tanh(s / softcap);",
     "if (softcap > 0.0) s = s;"),
    ("softcap_without_inner_division",
     "if (softcap > 0.0) s = softcap * tanh(s / softcap);",
     "if (softcap > 0.0) s = softcap * tanh(s);"),
    ("causal_ignored", "if (causal && j > qpos) return 0;",
     "if (causal && j > qpos + 1) return 0;"),
    ("no_normalisation", "out[d] = acc[d] / denom;", "out[d] = acc[d];"),
    ("max_sign_flipped", "double w = exp(x[j] - m);",
     "double w = exp(m - x[j]);"),
    ("value_from_wrong_head",
     "acc[d] += w * load_elem(v, (kv_head + j) * head_dim + d, fmt);",
     "acc[d] += w * load_elem(v, ((((int64_t)batch_idx * num_kv_heads + "
     "(hk + 1) % num_kv_heads) * kv_len) + j) * head_dim + d, fmt);"),
    ("empty_row_not_zero", "for (int d = 0; d < head_dim; ++d) out[d] = 0.0;",
     "for (int d = 0; d < head_dim; ++d) out[d] = 1.0;"),
    ("key_transposed_index",
     "load_elem(k, (kv_head + j) * head_dim + d, fmt);",
     "load_elem(k, kv_head * head_dim + (int64_t)d * kv_len + j, fmt);"),
    ("window_drops_current_key", "(qpos - j >= 0 &&", "(qpos - j > 0 &&"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mutant_is_caught(name, old, new, tmp_path):
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src.replace(old, new))
    lib = oracle.load(oracle.compile_oracle(str(path), str(tmp_path / f"{name}.so")))
    attn = c_oracle(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(attn)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
