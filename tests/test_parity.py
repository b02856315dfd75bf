"""CUDA path vs the fp64 oracle (GPU).

Bar: elementwise |gpu - oracle| <= 2e-2 + 2e-2 * |oracle| ("TPU v6e Masked
GQA Kernel Optimization", "Hard Constraints": rtol=2e-2, atol=2e-2 against an
fp32 reference; the oracle is fp64), no NaN anywhere, bitwise determinism run
to run ("Deterministic: same inputs, same output").  Every call goes through
the C ABI (``gqa_attn_fwd``) via the ctypes binding.
"""
import numpy as np
import pytest
import torch

import masked_grouped_query_b200 as mgq
from masked_grouped_query_b200.inputs import WORKLOADS, Workload, make_inputs
from oracle import oracle

RTOL = 2e-2
ATOL = 2e-2

pytestmark = pytest.mark.gpu


def run_gpu(w: Workload, q, k, v):
    out = mgq.attention(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, window=w.window,
                        softcap=w.softcap)
    torch.cuda.synchronize()
    return out


def assert_close(got: torch.Tensor, want: np.ndarray, what=""):
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - want)
    bound = ATOL + RTOL * np.abs(want)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; "
                           f"max err {err.max():.4g}")


def check_workload(w: Workload, q_scale=1.0, rows=None):
    q, k, v = make_inputs(w, q_scale=q_scale)
    out = run_gpu(w, q, k, v)
    if rows is None:
        want = oracle.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap)
        assert_close(out, want, w.name)
    else:
        want = oracle.attention_rows(q, k, v, causal=w.causal, window=w.window,
                                     softcap=w.softcap, rows=rows)
        assert_close(out.reshape(-1, w.head_dim)[torch.as_tensor(rows)], want, w.name)
    return q, k, v, out


# ---------------------------------------------------------- named workloads
@pytest.mark.parametrize("name", ["tiny_causal_gqa_prefill", "gqa_decode",
                                  "long_context_decode_16to1", "siglip_encoder",
                                  "long_window_softcap_prefill"])
def test_workload_full_output(name):
    # Every element of the full-size workload (the long window prefill costs
    # the oracle about 15 s on 8 cores).
    check_workload(WORKLOADS[name])


# ---------------------------------------------------------- shape sweep
SWEEP = [
    # (batch, q_len, kv_len, hq, hkv, d, causal, window, softcap)
    (1, 1, 1, 1, 1, 64, True, None, None),
    (2, 1, 130, 8, 2, 128, True, None, None),
    (1, 3, 200, 16, 1, 128, True, 50, 30.0),
    (2, 64, 64, 4, 4, 64, True, None, None),
    (1, 127, 300, 2, 1, 128, True, 17, None),
    (1, 129, 129, 4, 2, 128, False, None, 50.0),
    (2, 5, 3, 4, 2, 64, True, None, None),         # q_len > kv_len: empty rows
    (1, 40, 20, 6, 3, 80, True, 4, 10.0),          # empty rows + window
    (1, 17, 517, 16, 16, 72, False, None, None),   # D = 72, ragged
    (3, 9, 1000, 12, 4, 96, True, 128, None),
    (1, 2, 4099, 32, 2, 128, True, 1, None),       # window 1 = the diagonal key
    (1, 33, 77, 3, 1, 8, False, 5, 2.0),           # tiny head_dim
    (1, 6, 300, 4, 1, 256, True, None, 25.0),      # largest head_dim
    (2, 100, 180, 5, 5, 128, False, 64, None),     # window without causal
    (1, 8, 2048, 64, 4, 128, True, 4096, 30.0),    # window >= kv_len
]


@pytest.mark.parametrize("cfg", SWEEP, ids=[str(c) for c in SWEEP])
def test_shape_sweep(cfg):
    b, lq, lk, hq, hkv, d, causal, window, cap = cfg
    w = Workload("sweep", b, lq, lk, hq, hkv, d, causal, window, cap, seed=lq * 7 + lk)
    check_workload(w)


def test_empty_rows_are_zero_not_nan():
    w = Workload("e", 2, 12, 5, 8, 2, 128, True, None, 30.0, 5)
    q, k, v, out = check_workload(w)
    assert torch.all(out[:, :, :7] == 0)   # qpos = -7 .. -1 see nothing


@pytest.mark.parametrize("cfg", [(1, 300, 300, 4, 2, 128), (2, 200, 200, 2, 2, 72)])
def test_wide_logit_range_without_softcap(cfg):
    # q scaled by 30 and no softcap: scores spread over hundreds of log2
    # units, so on unmasked tiles many exponents fall far below the row max
    # (where the FMA-pipe 2^x clamps); the result must stay finite and match.
    b, lq, lk, hq, hkv, d = cfg
    check_workload(Workload("wide", b, lq, lk, hq, hkv, d, False, None, None, lq + d), q_scale=30.0)


@pytest.mark.parametrize("two_pass", [0, 1])
@pytest.mark.parametrize("cap,q_scale", [(5.0, 1.0), (50.0, 1.0), (50.0, 20.0), (63.0, 3.0),
                                         (64.0, 3.0), (200.0, 20.0)])
def test_softcap_fixed_base_and_row_max_paths_agree(cap, q_scale, two_pass):
    # Caps up to about 63.8 take one pass with a fixed exponent base (no row
    # max); larger caps, and every cap with the override set, find the row
    # max first.  Both must match the oracle on masked, ragged tiles, with
    # logits inside the polynomial's range (q_scale 1) and saturating ones
    # (q_scale 20, the hardware tanh).
    mgq.set_override("softcap_two_pass", two_pass)
    try:
        for w in (Workload("fb", 1, 300, 700, 8, 2, 128, True, 256, cap, 7),
                  Workload("fb2", 2, 129, 129, 4, 4, 72, False, None, cap, 8),
                  Workload("fb3", 1, 4, 3000, 64, 4, 128, True, 1000, cap, 9)):
            check_workload(w, q_scale=q_scale)
    finally:
        mgq.set_override("softcap_two_pass", 0)


def test_zero_kv_len_gives_zeros():
    q = torch.randn(2, 4, 3, 64, device="cuda").bfloat16()
    k = torch.empty(2, 2, 0, 64, device="cuda", dtype=torch.bfloat16)
    out = mgq.attention(q, k, k, causal=True)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_softcap_saturating_inputs():
    # q scaled by 20: raw logits reach ~|200|, far into tanh's flat region, so
    # a missing or misplaced softcap would be far outside tolerance.
    for cap in (30.0, 50.0, 5.0):
        w = Workload("sat", 2, 4, 600, 16, 4, 128, True, 256, cap, seed=int(cap))
        check_workload(w, q_scale=20.0)
        w2 = Workload("sat2", 1, 200, 200, 4, 1, 128, True, None, cap, seed=int(cap) + 1)
        check_workload(w2, q_scale=20.0)


def test_softcap_polynomial_degrees():
    # Caps up to 256 take the degree-5 tanh polynomial in the tcgen05
    # kernel, larger ones the degree-7 one; both against the oracle, with
    # q scaled so the logits span tens of units.
    for cap, seed in ((200.0, 41), (300.0, 42), (1000.0, 43)):
        w = Workload("capdeg", 1, 200, 300, 8, 2, 128, True, None, cap, seed=seed)
        assert mgq.describe(1, 200, 300, 8, 2, 128, True, None, cap)["path"] == "prefill"
        check_workload(w, q_scale=8.0)


def test_constant_v_returns_v():
    w = Workload("c", 2, 4, 700, 16, 4, 128, True, 300, 30.0, 8)
    q, k, _ = make_inputs(w)
    c = torch.randn(2, 4, 1, 128).bfloat16()
    v = c.expand(2, 4, 700, 128).contiguous()
    out = run_gpu(w, q, k, v).cpu()
    want = c.repeat_interleave(4, dim=1).expand_as(out)
    diff = (out.float() - want.float()).abs()
    ulp = want.float().abs() * 2.0 ** -7 + 1e-6   # one bf16 ulp
    assert torch.all(diff <= ulp)


def test_masked_keys_do_not_matter():
    # Keys outside every row's window: replace them with huge finite values.
    w = Workload("m", 2, 4, 900, 16, 4, 128, True, 200, None, 9)
    q, k, v = make_inputs(w)
    base = run_gpu(w, q, k, v).cpu()
    first_visible = 900 - 4 - 200 + 1  # qpos_min - window + 1
    k2, v2 = k.clone(), v.clone()
    k2[:, :, :first_visible] = 3.0e4
    v2[:, :, :first_visible] = -3.0e4
    got = run_gpu(w, q, k2, v2).cpu()
    assert torch.equal(base, got)


def test_gqa_equals_mha_on_gpu():
    w = Workload("g", 1, 3, 500, 16, 2, 128, True, None, 20.0, 12)
    q, k, v = make_inputs(w)
    a = run_gpu(w, q, k, v)
    wm = w.with_(num_kv_heads=16)
    m = run_gpu(wm, q, k.repeat_interleave(8, dim=1).contiguous(),
                v.repeat_interleave(8, dim=1).contiguous())
    want = oracle.attention(q, k, v, causal=True, window=None, softcap=20.0)
    assert_close(a, want, "gqa")
    assert_close(m, want, "mha")


@pytest.mark.parametrize("name", ["gqa_decode", "long_context_decode_16to1",
                                  "tiny_causal_gqa_prefill"])
def test_deterministic(name):
    w = WORKLOADS[name]
    q, k, v = make_inputs(w)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    a = mgq.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap)
    b = mgq.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("shape,splits", [
    ((16, 1, 8192, 32, 8, 128), 1),    # 128 units: one CTA per unit
    ((4, 1, 8192, 32, 8, 128), 5),     # 32 units: about one CTA per SM in total
    ((16, 1, 32768, 32, 8, 128), 4),   # no split longer than 128 key tiles
])
def test_decode_split_rule(shape, splits):
    # Single-token decode plans aim at about one CTA per SM (148 SMs on B200),
    # with no split longer than 128 key tiles of 64 keys.
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    plan = mgq.describe(*shape, True)
    assert plan["path"] == "decode"
    if sms == 148:
        assert plan["splits"] == splits, plan
    units = shape[0] * shape[4]
    assert plan["ctas"] == units * plan["splits"]
    assert -(-plan["tiles"] // plan["splits"]) <= 128 or plan["splits"] == 1


@pytest.mark.parametrize("tps", [1, 3, 7, 1000])
def test_forced_split_geometries_agree_with_oracle(tps):
    # The split-KV decode kernel, forced, at several split sizes.
    w = WORKLOADS["long_context_decode_16to1"].with_(batch=2)
    mgq.set_override("force_path", 1)
    mgq.set_override("tiles_per_split", tps)
    try:
        check_workload(w)
    finally:
        mgq.set_override("tiles_per_split", 0)
        mgq.set_override("force_path", 0)


@pytest.mark.parametrize("cfg", [
    (8, 4, 32768, 64, 4, 128, True, 4096, 30.0),   # the 16:1 long-context decode shape
    (2, 20, 3000, 8, 2, 128, True, None, None),     # 80 rows per kv head
    (1, 3, 1000, 16, 1, 72, False, 300, None),      # window without causal, D = 72
    (3, 2, 777, 32, 2, 64, True, None, 20.0),       # ragged keys, D = 64
    (1, 130, 4000, 2, 1, 128, True, None, 30.0),    # 3 row tiles: two-tile pairs, split
    (1, 700, 2500, 1, 1, 96, False, 900, None),     # 6 row tiles, window, D = 96
])
def test_tcgen05_key_splits(cfg):
    # Few row tiles: the tcgen05 kernel splits each tile pair's key range
    # and merges the partials; the plan must actually split.
    b, lq, lk, hq, hkv, d, causal, window, cap = cfg
    w = Workload("ks", b, lq, lk, hq, hkv, d, causal, window, cap, seed=lk + d)
    plan = mgq.describe(b, lq, lk, hq, hkv, d, causal, window, cap)
    assert plan["path"] == "prefill" and plan["splits"] > 1, plan
    check_workload(w)
    q, k, v = make_inputs(w)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    a = mgq.attention(q, k, v, causal=causal, window=window, softcap=cap)
    b2 = mgq.attention(q, k, v, causal=causal, window=window, softcap=cap)
    torch.cuda.synchronize()
    assert torch.equal(a, b2)  # deterministic merge order


@pytest.mark.parametrize("cfg", [
    (8, 4, 32768, 64, 4, 128, True, 4096, 30.0),   # 4 CTAs per unit
    (1, 3, 1000, 16, 1, 72, False, 300, None),     # 2 CTAs per unit, D = 72
    (3, 2, 777, 32, 2, 64, True, None, 20.0),      # 4 CTAs per unit, D = 64
    (40, 4, 1000, 16, 1, 128, True, None, None),   # 3 CTAs per unit: uneven column slices
])
def test_paired_split_merges(cfg):
    # Units with one row tile take two key splits per CTA; the partials
    # merge by all CTAs of the unit's cluster after the cluster barrier
    # (automatic) or by the last CTA to finish (forced).  Both against the
    # oracle, each deterministic, and the two within rounding of each other.
    b, lq, lk, hq, hkv, d, causal, window, cap = cfg
    w = Workload("pm", b, lq, lk, hq, hkv, d, causal, window, cap, seed=lk + 3 * d)
    q, k, v = make_inputs(w)
    want = oracle.attention(q, k, v, causal=causal, window=window, softcap=cap)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    outs = []
    try:
        for mode in (0, -1):
            mgq.set_override("prefill_cluster", mode)
            plan = mgq.describe(b, lq, lk, hq, hkv, d, causal, window, cap)
            # mode 0 must really take the cluster merge, mode -1 the workspace
            assert (plan["cluster"] >= 2) if mode == 0 else (plan["cluster"] == 0), plan
            a = mgq.attention(q, k, v, causal=causal, window=window, softcap=cap)
            a2 = mgq.attention(q, k, v, causal=causal, window=window, softcap=cap)
            torch.cuda.synchronize()
            assert torch.equal(a, a2)
            assert_close(a, want, f"merge mode {mode}")
            outs.append(a.float())
    finally:
        mgq.set_override("prefill_cluster", 0)
    assert (outs[0] - outs[1]).abs().max().item() <= 2.0 ** -6


def test_host_buffer_entry_point_matches_device_entry_point():
    w = Workload("h", 2, 3, 333, 8, 2, 128, True, 100, 30.0, 21)
    q, k, v = make_inputs(w)
    dev = run_gpu(w, q, k, v).cpu()
    qp, kp, vp = (t.pin_memory() for t in (q, k, v))
    host = mgq.attention_host(qp, kp, vp, causal=True, window=100, softcap=30.0)
    assert torch.equal(dev, host)


def test_clear_status_then_split_calls_match_oracle():
    # After a bounded wait has given up (the self test sets the status bit),
    # clear_status resets the word and every split ticket counter; split
    # calls on both kernels then match the oracle again.
    mgq.selftest_bounded_wait(1000)
    torch.cuda.synchronize()
    assert mgq.status() & 0x20
    mgq.clear_status()
    assert mgq.status() == 0
    for w in (WORKLOADS["gqa_decode"].with_(batch=2),
              Workload("cs", 1, 130, 4000, 2, 1, 128, True, None, 30.0, 77)):
        plan = mgq.describe(w.batch, w.q_len, w.kv_len, w.num_q_heads, w.num_kv_heads,
                            w.head_dim, w.causal, w.window, w.softcap)
        assert plan["splits"] > 1 and plan["cluster"] == 0, plan
        check_workload(w)
    assert mgq.status() == 0


def test_no_bounded_wait_expired():
    torch.cuda.synchronize()
    assert mgq.status() & 0x1f == 0


@pytest.mark.parametrize("tiles,splits", [(8, 6), (11, 8)])
@pytest.mark.parametrize("merge", [0, -1])
def test_uneven_paired_splits(tiles, splits, merge):
    # Split s of S takes key tiles [ceil(s T / S), ceil((s + 1) T / S)).  For
    # these (T, S) some paired item's second split is the larger one (8 in 6:
    # sizes 2 1 | 1 2 | 1 1), so its tile A takes that split instead.  Both
    # merges (cluster, and last CTA with key 4 = -1) against the oracle.
    w = Workload("us", 2, 4, tiles * 128, 16, 1, 128, False, None, None, seed=10 * tiles + splits)
    q, k, v = make_inputs(w)
    want = oracle.attention(q, k, v, causal=False, window=None, softcap=None)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    try:
        mgq.set_override("prefill_splits", splits)
        mgq.set_override("prefill_cluster", merge)
        plan = mgq.describe(2, 4, tiles * 128, 16, 1, 128)
        assert plan["path"] == "prefill" and plan["splits"] == splits and plan["tiles"] == tiles, plan
        assert (plan["cluster"] >= 2) if merge == 0 else (plan["cluster"] == 0), plan
        a = mgq.attention(q, k, v)
        torch.cuda.synchronize()
        assert_close(a, want, f"{tiles} tiles in {splits} splits, merge {merge}")
    finally:
        mgq.set_override("prefill_splits", 0)
        mgq.set_override("prefill_cluster", 0)
