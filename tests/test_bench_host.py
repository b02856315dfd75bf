"""Host logic of bench.py (CPU): the algorithmic work each workload is
measured against, and the kernel-source hash that keeps committed ncu
figures tied to the code they were taken on."""
import os
import shutil

import pytest

import bench
from masked_grouped_query_b200.inputs import WORKLOADS


def test_work_counts_match_closed_forms():
    # tiny causal prefill, Lq = Lk = 128: row i sees keys 0..i.
    assert bench.visible_pairs_per_head(WORKLOADS["tiny_causal_gqa_prefill"]) == 128 * 129 // 2
    # causal window W = 1024 over Lq = Lk = 4096: min(i + 1, W) keys per row.
    w = WORKLOADS["long_window_softcap_prefill"]
    want = sum(min(i + 1, 1024) for i in range(4096))
    assert bench.visible_pairs_per_head(w) == want == 3_670_528
    # encoder: no mask, every pair.
    assert bench.visible_pairs_per_head(WORKLOADS["siglip_encoder"]) == 729 * 729
    # single-token causal decode: the whole cache, K and V, bf16.
    w = WORKLOADS["gqa_decode"]
    assert bench.kv_union_keys(w) == 8192
    assert bench.kv_bytes(w) == 2 * 2 * 128 * 8192 * 16 * 8
    # 4 query positions 32764..32767, window 4096: keys 28669..32767.
    w = WORKLOADS["long_context_decode_16to1"]
    assert bench.kv_union_keys(w) == 32767 - (32764 - 4095) + 1 == 4099
    assert bench.kv_bytes(w) == 2 * 2 * 128 * 4099 * 8 * 4


def test_decode_class():
    assert bench.is_decode(WORKLOADS["gqa_decode"])
    assert bench.is_decode(WORKLOADS["long_context_decode_16to1"])   # 16 heads x 4 rows
    assert not bench.is_decode(WORKLOADS["tiny_causal_gqa_prefill"])
    assert not bench.is_decode(WORKLOADS["siglip_encoder"])


def test_strip_comments_keeps_code_and_strings():
    src = 'asm("a // not a comment"); // gone\n/* gone\n too */ int x = 1;  \n'
    assert bench._strip_comments(src) == 'asm("a // not a comment"); int x = 1;'


def test_source_hash_ignores_comments_only(tmp_path):
    csrc = os.path.join(bench.ROOT, "masked_grouped_query_b200", "csrc")
    copy = tmp_path / "csrc"
    shutil.copytree(csrc, copy)
    base = bench.kernel_source_hash(str(copy))
    assert base == bench.kernel_source_hash()
    f = copy / "mask.cuh"
    text = f.read_text()
    f.write_text("// a new comment line\n" + text.replace("\n", "  \n", 3))
    assert bench.kernel_source_hash(str(copy)) == base
    f.write_text(text + "\nstatic const int kHashProbe = 1;\n")
    assert bench.kernel_source_hash(str(copy)) != base


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_metric_units(name):
    metric, unit, work = bench.metric_of(WORKLOADS[name])
    assert unit in ("GB/s", "TFLOP/s") and work > 0
