"""The KV-cache update oracle against its pins (CPU), with planted controls:
each mutant of the oracle's source must fail at least one pin."""
import importlib.util

import numpy as np
import pytest

from oracle import kv_cache

from . import kv_cache_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=[p.__name__ for p in pins.ALL_PINS])
def test_kv_oracle_pins(pin):
    pin(kv_cache)


def test_kv_oracle_rejects_blocks_that_do_not_fit():
    k = np.zeros((1, 4, 1, 2), np.float32)
    new = np.zeros((1, 2, 1, 2), np.float32)
    for pos in (-1, 3, 4):
        with pytest.raises(ValueError):
            kv_cache.kv_update(k, k, new, new, pos)
    with pytest.raises(ValueError):
        kv_cache.kv_update(k, k, np.zeros((1, 2, 2, 2), np.float32), new, 0)


MUTANTS = [
    ("slot_off_by_one", "kc[:, position:position + length] = convert(new_keys, cache_dtype)",
     "kc[:, position + 1:position + length + 1] = convert(new_keys, cache_dtype)"),
    ("values_into_key_cache",
     "vc[:, position:position + length] = convert(new_values, cache_dtype)",
     "kc[:, position:position + length] = convert(new_values, cache_dtype)"),
    ("ties_always_up", "round_up = (lower > half) | ((lower == half) & ((upper & 1) == 1))",
     "round_up = lower >= half"),
    ("truncation", "out = (upper + round_up.astype(np.uint64)) & 0xFFFF",
     "out = upper & 0xFFFF"),
    ("ties_to_odd", "((upper & 1) == 1)", "((upper & 1) == 0)"),
    ("length_without_position",
     "vc[:, position:position + length] = convert(new_values, cache_dtype)\n    return kc, vc, position + length",
     "vc[:, position:position + length] = convert(new_values, cache_dtype)\n    return kc, vc, length"),
    ("ring_length_without_position", "        vc[:, slot] = nv[:, i]\n    return kc, vc, position + length",
     "        vc[:, slot] = nv[:, i]\n    return kc, vc, length"),
    ("widening_shift", "(b.astype(np.uint32) << 16)", "(b.astype(np.uint32) << 15)"),
    ("ring_slot_off_by_one", "        slot = (position + i) % s", "        slot = (position + i + 1) % s"),
    ("ring_read_back_shifted", "        out[:, j] = ring[:, j % s]", "        out[:, j] = ring[:, (j + 1) % s]"),
    ("ring_keeps_one_too_few", "    for j in range(max(0, kv_len - s), kv_len):",
     "    for j in range(max(0, kv_len - s + 1), kv_len):"),
    ("no_conversion_for_bf16", "return new.copy() if new.dtype == np.uint16 else "
     "f32_to_bf16_bits(new)", "return new.copy() if new.dtype == np.uint16 else "
     "(new.view(np.uint32) >> 16).astype(np.uint16)"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_kv_mutant_is_caught(name, old, new, tmp_path):
    src = open(kv_cache.__file__).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    path = tmp_path / f"kv_mut_{name}.py"
    path.write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"kv_mut_{name}", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(mod)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
