#!/usr/bin/env python
"""Benchmark of the masked GQA attention forward pass (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl {native,reference}] [--all]

A step is one call of ``gqa_attn_fwd`` over one batch of the workload -- the
whole hot path (validate/plan, the attention kernel with its fused split-KV
combine).  Inputs are seeded synthetic bf16 N(0,1) of the workload's shape,
resident in HBM before timing; between timed steps L2 is flushed (a 256 MiB
buffer written, then read back, so no dirty line of the flush is written back
inside the timed kernel), and each step is timed with CUDA events on the
launching stream.

Metric: decode workloads report K/V-read GB/s -- bytes of the keys in the
union of the visible ranges, read once per kv head -- and prefill/encoder
workloads report TFLOP/s over unmasked (q, k) pairs at 4 * head_dim FLOP per
pair; both are compared with the measured peaks of the box.

``--impl reference`` times the fp64 CPU oracle (the slow reference arm) on a
bounded sample of the same workload.  Under torchrun (N > 1) each rank runs
its own replica (independent problems, no data-path collective: weak
scaling); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from masked_grouped_query_b200.inputs import (CACHE_STEPS, RING_STEPS, WORKLOADS,  # noqa: E402
                                              CacheStep, Workload, make_inputs)

DEFAULT_WORKLOAD = "gqa_decode"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ------------------------------------------------------------ work counts
def is_decode(w: Workload) -> bool:
    """Decode-class workloads (few query rows per kv head) are HBM-bound."""
    return w.group * w.q_len <= 64


def _first_last(w: Workload, qpos: np.ndarray):
    first = np.zeros_like(qpos)
    last = np.full_like(qpos, w.kv_len - 1)
    if w.window:
        first = np.maximum(0, qpos - w.window + 1)
    if w.causal or w.window:
        last = np.minimum(w.kv_len - 1, qpos)
    return first, last


def visible_pairs_per_head(w: Workload) -> int:
    qpos = (w.kv_len - w.q_len) + np.arange(w.q_len, dtype=np.int64)
    first, last = _first_last(w, qpos)
    return int(np.maximum(0, last - first + 1).sum())


def useful_flops(w: Workload) -> float:
    """4 * D FLOP per unmasked (q, k) pair, logical head_dim."""
    return 4.0 * w.head_dim * visible_pairs_per_head(w) * w.batch * w.num_q_heads


def kv_union_keys(w: Workload) -> int:
    qpos = (w.kv_len - w.q_len) + np.arange(w.q_len, dtype=np.int64)
    first, last = _first_last(w, qpos)
    ok = last >= first
    if not ok.any():
        return 0
    return int(last[ok].max() - first[ok].min() + 1)


def kv_bytes(w: Workload) -> float:
    """K and V bytes of the visible key union, read once per kv head."""
    return 2.0 * 2 * w.head_dim * kv_union_keys(w) * w.batch * w.num_kv_heads


def metric_of(w: Workload):
    if is_decode(w):
        return ("masked-GQA attn fwd KV-read GB/s (decode)", "GB/s", kv_bytes(w) / 1e9)
    return ("masked-GQA attn fwd TFLOP/s (prefill)", "TFLOP/s", useful_flops(w) / 1e12)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


_CODE_TOKENS = re.compile(r'"(?:\\.|[^"\\\n])*"|(?:\s|//[^\n]*|/\*.*?\*/)+', re.S)


def _strip_comments(text: str) -> str:
    """C/CUDA source with comments removed and whitespace runs collapsed
    (string literals kept), so edits to comments alone keep the hash."""
    def sub(m):
        t = m.group(0)
        return t if t.startswith('"') else " "
    return _CODE_TOKENS.sub(sub, text).strip()


def kernel_source_hash(csrc: str | None = None) -> str:
    """Hash of the kernel sources' code (not their comments): the ncu figures
    in profiles/traffic.json are reported only while it matches."""
    h = hashlib.sha256()
    csrc = csrc or os.path.join(ROOT, "masked_grouped_query_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), encoding="utf-8") as f:
                code = _strip_comments(f.read())
            h.update(name.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if still current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(workload)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def roofline_block(w: Workload, ms_mean: float, pk: dict, pk_src: str) -> dict:
    """Roofline of one attention workload timed at ``ms_mean`` ms per call:
    HBM for decode-class workloads (algorithmic K/V bytes), bf16 tensor peak
    otherwise (FLOPs over unmasked pairs)."""
    _, unit, work = metric_of(w)
    if unit == "GB/s":
        bound, peak = "hbm", pk["hbm_gbs"]
    else:
        bound, peak = "tensor", pk["bf16_tflops"]
    achieved = work / (ms_mean * 1e-3)
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak,
            "peak_source": f"{pk_src} (MEASURED_PEAKS.json)" if pk_src == "measured" else "fallback",
            "traffic": ncu_traffic(w.name)}


def workload_entry(w: Workload, res: dict, pk: dict, pk_src: str) -> dict:
    """One attention workload's figures from a timing result of _timed_loop."""
    name, unit, work = metric_of(w)
    return {"metric": name, "value": work / (res["ms_mean"] * 1e-3), "unit": unit,
            "ms_mean": res["ms_mean"], "ms_median": res["ms_median"],
            "ms_p10": res["ms_p10"], "ms_p90": res["ms_p90"],
            "config": {k: v for k, v in w.cfg().items() if k != "name"},
            "roofline": roofline_block(w, res["ms_mean"], pk, pk_src),
            "gpu_launches": res.get("launches"), "plan": res.get("plan"),
            "device_status": res.get("status")}


def other_workloads(main_name: str, timer, pk: dict, pk_src: str) -> dict:
    """Every attention workload except ``main_name``, each timed by
    ``timer(w)`` (the same L2 flush and CUDA-event timing as the headline)."""
    return {w.name: workload_entry(w, timer(w), pk, pk_src)
            for w in WORKLOADS.values() if w.name != main_name}


# ------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz)}


# ------------------------------------------------------------ native arm
def _timed_loop(call, steps: int, warmup: int, device, dist_ctx):
    """Run ``call`` warmup + steps times with an L2 flush before each; time
    each timed call with CUDA events on the current stream."""
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    sink = torch.empty((), dtype=torch.float32, device=device)

    def flush_l2():
        # Write a buffer twice the L2 size, then read it back: the inputs are
        # evicted and the L2 is left holding clean lines, so no write-back of
        # the flush itself lands inside the timed kernel.
        flush.fill_(0.0)
        torch.sum(flush, dim=0, out=sink)

    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        flush_l2()
        call()
    torch.cuda.synchronize(device)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    dist_ctx.barrier()
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    for i in range(steps):
        flush_l2()
        starts[i].record(stream)
        call()
        ends[i].record(stream)
    torch.cuda.synchronize(device)
    wall = time.perf_counter() - t0
    dist_ctx.barrier()
    per = [st.elapsed_time(en) for st, en in zip(starts, ends)]
    return {"ms_mean": float(np.mean(per)), "ms_median": float(np.median(per)),
            "ms_p10": float(np.percentile(per, 10)), "ms_p90": float(np.percentile(per, 90)),
            "wall_s": wall}


def time_native(w: Workload, steps: int, warmup: int, device, dist_ctx):
    import ctypes

    import masked_grouped_query_b200 as mgq
    from masked_grouped_query_b200 import _lib

    lib = _lib.load()
    q, k, v = (t.to(device) for t in make_inputs(w))
    out = torch.empty_like(q)
    sp = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    causal, window, cap = int(w.causal), int(w.window or 0), float(w.softcap or 0.0)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), w.batch, w.q_len,
            w.kv_len, w.num_q_heads, w.num_kv_heads, w.head_dim, causal, window, cap)

    def call():
        rc = lib.gqa_attn_fwd(*args, sp)
        if rc != 0:
            raise RuntimeError(f"gqa_attn_fwd: {_lib.error_string(rc)}")

    res = _timed_loop(call, steps, warmup, device, dist_ctx)
    res["launches"] = steps
    res["plan"] = mgq.describe(w.batch, w.q_len, w.kv_len, w.num_q_heads, w.num_kv_heads,
                               w.head_dim, w.causal, w.window, w.softcap)
    res["status"] = mgq.status()
    return res


def time_cache_step(st: CacheStep, steps: int, warmup: int, device, dist_ctx):
    """One decode step on a (batch, slots, heads, head_dim) bf16 cache: the
    fp32 new token is appended at ``position`` and attended with the rest,
    through ``gqa_attn_decode_append`` (one fused launch on the split-KV
    kernel).  Bytes: the attention's K/V union plus the append's fp32 reads
    and bf16 writes."""
    import ctypes

    from masked_grouped_query_b200 import _lib
    from masked_grouped_query_b200.inputs import make_cache_inputs

    lib = _lib.load()
    x = make_cache_inputs(st.batch, st.slots, st.num_kv_heads, st.head_dim, st.count,
                          seed=st.seed, num_q_heads=st.num_q_heads, device=device)
    out = torch.empty_like(x["q"])
    sp = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    args = (x["q"].data_ptr(), x["k_cache"].data_ptr(), x["v_cache"].data_ptr(),
            x["new_k"].data_ptr(), x["new_v"].data_ptr(), out.data_ptr(), st.batch, st.count,
            st.position, st.slots, st.num_q_heads, st.num_kv_heads, st.head_dim,
            0x1, int(st.causal), int(st.window or 0), float(st.softcap or 0.0), sp)

    def call():
        rc = lib.gqa_attn_decode_append(*args)
        if rc != 0:
            raise RuntimeError(f"gqa_attn_decode_append: {_lib.error_string(rc)}")

    res = _timed_loop(call, steps, warmup, device, dist_ctx)
    w = Workload(st.name, st.batch, st.count, st.kv_len, st.num_q_heads, st.num_kv_heads,
                 st.head_dim, st.causal, st.window, st.softcap, st.seed)
    append_bytes = 2.0 * st.batch * st.count * st.num_kv_heads * st.head_dim * (4 + 2)
    res["bytes"] = kv_bytes(w) + append_bytes
    return res


def time_ring(rs: dict, steps: int, warmup: int, device):
    """gqa_attn_fwd_ring on a (batch, kv_heads, slots, head_dim) ring: bytes
    are the K/V of the window's keys, read once per kv head."""
    import ctypes

    from masked_grouped_query_b200 import _lib

    lib = _lib.load()
    g = torch.Generator(device=device).manual_seed(rs["seed"])
    ks = (rs["batch"], rs["num_kv_heads"], rs["slots"], rs["head_dim"])
    kr = torch.randn(ks, generator=g, device=device).bfloat16()
    vr = torch.randn(ks, generator=g, device=device).bfloat16()
    q = torch.randn(rs["batch"], rs["num_q_heads"], rs["q_len"], rs["head_dim"], generator=g,
                    device=device).bfloat16()
    out = torch.empty_like(q)
    sp = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    args = (q.data_ptr(), kr.data_ptr(), vr.data_ptr(), out.data_ptr(), rs["batch"], rs["q_len"],
            rs["kv_len"], rs["slots"], rs["num_q_heads"], rs["num_kv_heads"], rs["head_dim"], 0,
            int(rs["causal"]), int(rs["window"] or 0), float(rs["softcap"] or 0.0), sp)

    def call():
        rc = lib.gqa_attn_fwd_ring(*args)
        if rc != 0:
            raise RuntimeError(f"gqa_attn_fwd_ring: {_lib.error_string(rc)}")

    res = _timed_loop(call, steps, warmup, device, _NoDist())
    w = Workload("ring", rs["batch"], rs["q_len"], rs["kv_len"], rs["num_q_heads"],
                 rs["num_kv_heads"], rs["head_dim"], rs["causal"], rs["window"], rs["softcap"],
                 rs["seed"])
    res["bytes"] = kv_bytes(w)
    return res


def time_kv_append(batch: int, count: int, heads: int, head_dim: int, slots: int, steps: int,
                   warmup: int, device):
    """The append kernel alone on a prompt-sized block (fp32 tokens into a
    bf16 (batch, slots, heads, head_dim) cache): bytes read + written."""
    import ctypes

    from masked_grouped_query_b200 import _lib
    from masked_grouped_query_b200.inputs import make_cache_inputs

    lib = _lib.load()
    x = make_cache_inputs(batch, slots, heads, head_dim, count, seed=17, device=device)
    sp = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    args = (x["k_cache"].data_ptr(), x["v_cache"].data_ptr(), x["new_k"].data_ptr(),
            x["new_v"].data_ptr(), batch, slots, heads, head_dim, 0, count, 0x1, None, sp)

    def call():
        rc = lib.gqa_attn_kv_append(*args)
        if rc != 0:
            raise RuntimeError(f"gqa_attn_kv_append: {_lib.error_string(rc)}")

    res = _timed_loop(call, steps, warmup, device, _NoDist())
    res["bytes"] = 2.0 * batch * count * heads * head_dim * (4 + 2)
    return res


def time_e2e(w: Workload, steps: int, warmup: int, device):
    """Same metric through the host-buffer C call: H2D, kernel, D2H per step."""
    from masked_grouped_query_b200 import _lib
    import ctypes

    lib = _lib.load()
    qh, kh, vh = (t.pin_memory() for t in make_inputs(w))
    oh = torch.empty(qh.shape, dtype=qh.dtype, pin_memory=True)
    dq, dk, dv = (torch.empty(t.shape, dtype=t.dtype, device=device) for t in (qh, kh, vh))
    do = torch.empty_like(dq)
    sp = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    args = (qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), oh.data_ptr(), dq.data_ptr(),
            dk.data_ptr(), dv.data_ptr(), do.data_ptr(), w.batch, w.q_len, w.kv_len,
            w.num_q_heads, w.num_kv_heads, w.head_dim, int(w.causal), int(w.window or 0),
            float(w.softcap or 0.0), sp)
    for _ in range(warmup):
        rc = lib.gqa_attn_fwd_host(*args)
        if rc != 0:
            raise RuntimeError(f"gqa_attn_fwd_host: {_lib.error_string(rc)}")
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        rc = lib.gqa_attn_fwd_host(*args)
        if rc != 0:
            raise RuntimeError(f"gqa_attn_fwd_host: {_lib.error_string(rc)}")
    e.record(stream)
    torch.cuda.synchronize(device)
    ms = s.elapsed_time(e) / steps
    h2d = (qh.numel() + kh.numel() + vh.numel()) * 2
    return ms, h2d, oh.numel() * 2


# ------------------------------------------------------------ oracle arm
def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "" when unknown."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return ""


def cpu_sample(w: Workload, budget_s: float = 12.0):
    """Time the oracle on whole kv-head groups of the workload; returns
    (metric value, sample description, threads, seconds)."""
    from oracle import oracle

    q, k, v = make_inputs(w)
    threads = len(os.sched_getaffinity(0))
    units = w.batch * w.num_kv_heads
    g = w.group
    name, unit, work = metric_of(w)
    per_unit_work = work / units
    # first a single kv-head group to size the sample
    # Whole groups, cycling through the workload until the time budget is
    # spent (a workload smaller than the budget is computed several times).
    n_units, elapsed, done = 1, 0.0, 0
    rows_per_unit = g * w.q_len
    while True:
        ids = []
        for u in range(done, done + min(n_units, units)):
            b, kvh = divmod(u % units, w.num_kv_heads)
            for h in range(kvh * g, (kvh + 1) * g):
                base = (b * w.num_q_heads + h) * w.q_len
                ids.extend(range(base, base + w.q_len))
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap,
                              rows=np.asarray(ids, dtype=np.int64), threads=threads)
        dt = time.perf_counter() - t0
        got = len(ids) // rows_per_unit
        done += got
        elapsed += dt
        if elapsed >= budget_s:
            break
        n_units = max(1, int(got * max(1.0, (budget_s - elapsed) / max(dt, 1e-6))))
    value = per_unit_work * done / elapsed
    desc = (f"{done} (batch, kv head) groups of {units} in the workload "
            f"({done * rows_per_unit} query rows; {done / units:.2f} passes), fp64 oracle, "
            f"{elapsed:.1f} s")
    return value, desc, threads, elapsed


# ------------------------------------------------------------ distributed
class DistCtx:
    def __init__(self, n_gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            torch.cuda.set_device(self.local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", self.local))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch.distributed as dist
        t = torch.tensor([x], dtype=torch.float64, device=f"cuda:{self.local}")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    choices=list(WORKLOADS) + list(EXTRA_WORKLOADS),
                    help="an attention workload, or one of the KV-cache / ring extras "
                         "(timed alone: one JSON line with its roofline, 1 GPU)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--all", action="store_true",
                    help="also time the KV-cache, ring-window and append extras")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the other attention workloads (timed by default at N = 1)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.workload in EXTRA_WORKLOADS:
        if args.impl == "reference":
            if int(os.environ.get("RANK", "0")) == 0:
                print(json.dumps({"impl": "reference", "unavailable":
                                  "the oracle arm times the attention workloads only"}))
            return
        return run_extra(args)
    w = WORKLOADS[args.workload]
    name, unit, work = metric_of(w)
    pk, pk_src = peaks()

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return
        vals = []
        desc = threads = None
        for _ in range(args.warmup):
            pass  # the oracle has nothing to warm up beyond the first call below
        budget = max(1.0, 60.0 / max(1, args.steps))
        for _ in range(args.steps):
            val, desc, threads, _ = cpu_sample(w, budget_s=budget)
            vals.append(val)
        value = float(np.median(vals))
        line = {"impl": "reference", "metric": name, "value": value, "unit": unit,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": work / value * 1e3 if value else None,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f64", "data": "synthetic",
                "config": {"workload": w.name, **{k: v for k, v in w.cfg().items() if k not in ("name",)}},
                "cpu_baseline": {"value": value, "unit": unit, "cores": threads,
                                 "kind": "oracle", "sample": desc, "cpu": cpu_model()},
                "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    ctx = DistCtx(args.gpus)
    device = torch.device("cuda", ctx.local)
    torch.cuda.set_device(device)
    from masked_grouped_query_b200 import build as _build
    if not os.path.exists(_build.LIBRARY):
        raise SystemExit("libgqa_attn.so missing: run __graft_entry__.build() first")

    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(ctx.local)).split(",")[ctx.local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else ctx.local
    with ClockSampler(gpu_index) as clk:
        res = time_native(w, args.steps, args.warmup, device, ctx)
        e2e = None
        if not args.no_e2e:
            e2e_steps = max(3, min(args.steps, 20))
            e2e = time_e2e(w, e2e_steps, 3, device)
    ms = ctx.max(res["ms_mean"])
    value = work * ctx.world / (ms * 1e-3)

    extra = {}
    others_clocks = None
    if ctx.world == 1 and not args.no_others:
        # The other configurations of the metric, each timed like the headline.
        with ClockSampler(gpu_index) as clk2:
            extra = other_workloads(
                w.name, lambda o: time_native(o, args.steps, args.warmup, device, _NoDist()),
                pk, pk_src)
        others_clocks = clk2.summary()
    if args.all and ctx.rank == 0:
        for st in CACHE_STEPS.values():
            r = time_cache_step(st, max(20, args.steps // 4), args.warmup, device, _NoDist())
            a = r["bytes"] / 1e9 / (r["ms_mean"] * 1e-3)
            extra[st.name] = {"metric": "decode step on a KV cache (append + attend) GB/s",
                              "value": a, "unit": "GB/s", "ms": r["ms_mean"],
                              "frac_of_peak": a / pk["hbm_gbs"], "launches_per_step": 1}
        for ring_name, rs in RING_STEPS.items():
            r = time_ring(rs, max(20, args.steps // 4), args.warmup, device)
            a = r["bytes"] / 1e9 / (r["ms_mean"] * 1e-3)
            extra[ring_name] = {"metric": "masked-GQA attn fwd KV-read GB/s (decode, ring window)",
                                "value": a, "unit": "GB/s", "ms": r["ms_mean"],
                                "frac_of_peak": a / pk["hbm_gbs"],
                                "shape": {k: v for k, v in rs.items() if k != "seed"}}
        r = time_kv_append(2, 4096, 4, 128, 4096, max(20, args.steps // 4), args.warmup, device)
        a = r["bytes"] / 1e9 / (r["ms_mean"] * 1e-3)
        extra["kv_append_prompt_block"] = {
            "metric": "KV-cache append GB/s (fp32 in, bf16 cache, read + written bytes)",
            "value": a, "unit": "GB/s", "ms": r["ms_mean"], "frac_of_peak": a / pk["hbm_gbs"],
            "shape": "batch 2, 4096 tokens, 4 kv heads, head_dim 128, (B,S,H,D) cache"}

    if ctx.rank == 0:
        roof = roofline_block(w, res["ms_mean"], pk, pk_src)
        line = {"metric": name, "value": value, "unit": unit, "n_gpus": ctx.world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": w.name,
                           **{k: v for k, v in w.cfg().items() if k not in ("name",)},
                           "l2": "flushed between timed steps (256 MiB write, then read)",
                           "parallelism": f"replica x{ctx.world}"},
                "roofline": roof,
                "gpu_launches": res["launches"],
                "plan": res["plan"], "device_status": res["status"],
                "ms_median": res["ms_median"], "ms_p10": res["ms_p10"], "ms_p90": res["ms_p90"],
                "clocks": clk.summary()}
        if e2e is not None:
            ms_e2e, h2d, d2h = e2e
            line["e2e"] = {"value": work / (ms_e2e * 1e-3), "unit": unit,
                           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                           "ms_per_step": ms_e2e}
        if ctx.world == 1 and not args.no_cpu:
            val, desc, threads, _ = cpu_sample(w)
            line["cpu_baseline"] = {"value": val, "unit": unit, "cores": threads,
                                    "kind": "oracle", "sample": desc, "cpu": cpu_model()}
        if extra:
            line["other_workloads"] = extra
        if others_clocks is not None:
            line["other_workloads_clocks"] = others_clocks
        print(json.dumps(line))
    ctx.close()


EXTRA_WORKLOADS = ("gqa_decode_append", "gqa_decode_ring_window", "kv_append_prompt_block")


def run_extra(args):
    """Time one of the extras alone on GPU 0 and print its line (HBM roofline)."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    pk, pk_src = peaks()
    name = args.workload
    with ClockSampler(0) as clk:
        if name in CACHE_STEPS:
            r = time_cache_step(CACHE_STEPS[name], args.steps, args.warmup, device, _NoDist())
            metric, launches = "decode step on a KV cache (append + attend) GB/s", 1
            cfg = {k: v for k, v in vars(CACHE_STEPS[name]).items() if k != "seed"}
        elif name in RING_STEPS:
            r = time_ring(RING_STEPS[name], args.steps, args.warmup, device)
            metric, launches = "masked-GQA attn fwd KV-read GB/s (decode, ring window)", 1
            cfg = {k: v for k, v in RING_STEPS[name].items() if k != "seed"}
        else:
            r = time_kv_append(2, 4096, 4, 128, 4096, args.steps, args.warmup, device)
            metric, launches = "KV-cache append GB/s (fp32 in, bf16 cache, read + written bytes)", 1
            cfg = {"batch": 2, "tokens": 4096, "kv_heads": 4, "head_dim": 128, "slots": 4096,
                   "cache": "(B,S,H,D) bf16", "new": "(B,L,H,D) fp32"}
    value = r["bytes"] / 1e9 / (r["ms_mean"] * 1e-3)
    roof = {"bound": "hbm", "achieved": value, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": value / pk["hbm_gbs"],
            "peak_source": f"{pk_src} (MEASURED_PEAKS.json)" if pk_src == "measured" else "fallback",
            "traffic": ncu_traffic(name)}
    line = {"metric": metric, "value": value, "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_mean"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": name, **cfg,
                       "l2": "flushed between timed steps (256 MiB write, then read)"},
            "roofline": roof, "gpu_launches": launches * args.steps, "clocks": clk.summary()}
    print(json.dumps(line))


class _NoDist:
    def barrier(self):
        pass


if __name__ == "__main__":
    main()
