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


def test_default_run_reports_every_other_config_with_its_roofline():
    # The headline is one workload; the other four configurations of the
    # metric come with the same timing fields and a roofline block each.
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0}
    seen = []

    def timer(w):  # stands in for the CUDA-event loop
        seen.append(w.name)
        return {"ms_mean": 0.1, "ms_median": 0.09, "ms_p10": 0.08, "ms_p90": 0.12,
                "launches": 20, "plan": {"path": 2}, "status": 0}

    out = bench.other_workloads("gqa_decode", timer, pk, "fallback")
    assert sorted(out) == sorted(n for n in WORKLOADS if n != "gqa_decode") == sorted(seen)
    for name, e in out.items():
        w = WORKLOADS[name]
        _, unit, work = bench.metric_of(w)
        roof = e["roofline"]
        assert e["unit"] == roof["unit"] == unit
        assert roof["bound"] == ("hbm" if unit == "GB/s" else "tensor")
        assert roof["peak"] == (pk["hbm_gbs"] if unit == "GB/s" else pk["bf16_tflops"])
        assert abs(roof["achieved"] - work / 1e-4) < 1e-6 * roof["achieved"]
        assert abs(roof["frac"] - roof["achieved"] / roof["peak"]) < 1e-12
        assert e["value"] == roof["achieved"]
        assert e["ms_median"] == 0.09 and e["gpu_launches"] == 20
        assert "traffic" in roof
