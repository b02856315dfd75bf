"""KV-cache append and the decode step on a cache: CUDA path vs the oracles (GPU).

The append is data movement plus one rounding, so the bar is bit-exact
against ``oracle.kv_cache`` (NaN compared as NaN: its payload is not fixed).
The attention after the append uses the attention bar of ``test_parity``
against the fp64 oracle run on the oracle-updated cache, and must equal, bit
for bit, ``gqa_attn_fwd`` on a contiguous copy of the filled slots.
"""
import numpy as np
import pytest
import torch

import masked_grouped_query_b200 as mgq
from masked_grouped_query_b200 import _lib
from masked_grouped_query_b200.inputs import CACHE_STEPS, make_cache_inputs
from oracle import kv_cache as okv
from oracle import oracle

from .test_parity import assert_close

pytestmark = pytest.mark.gpu


def bits_of(t: torch.Tensor) -> np.ndarray:
    """Host numpy view in the oracle's representation (bf16 -> uint16 bits)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bf16_from_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def to_layout(t: torch.Tensor, head_major: bool) -> torch.Tensor:
    """(B, S|L, H, D) page layout -> head-major (B, H, S|L, D) when asked."""
    return t.transpose(1, 2).contiguous() if head_major else t.contiguous()


def from_layout(t: torch.Tensor, head_major: bool) -> torch.Tensor:
    return t.transpose(1, 2).contiguous() if head_major else t


def assert_same_bits(got: np.ndarray, want: np.ndarray, what: str):
    assert got.shape == want.shape and got.dtype == want.dtype, what
    if got.dtype == np.uint16:
        gnan = np.isnan(okv.bf16_bits_to_f32(got))
        wnan = np.isnan(okv.bf16_bits_to_f32(want))
    else:
        gnan, wnan = np.isnan(got), np.isnan(want)
    assert np.array_equal(gnan, wnan), f"{what}: NaN positions differ"
    g = got.view(np.uint32 if got.dtype == np.float32 else np.uint16)
    w = want.view(g.dtype)
    bad = (g != w) & ~gnan
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} elements differ"


COMBOS = [(cache_dt, new_dt, seq_major, new_hm)
          for cache_dt in (torch.bfloat16, torch.float32)
          for new_dt in (torch.float32, torch.bfloat16)
          for seq_major in (True, False)
          for new_hm in (False, True)]


@pytest.mark.parametrize("combo", COMBOS, ids=[
    f"{str(c[0])[6:]}-new_{str(c[1])[6:]}-{'seq' if c[2] else 'head'}-"
    f"{'newhm' if c[3] else 'newseq'}" for c in COMBOS])
@pytest.mark.parametrize("shape", [(2, 37, 3, 64, 5, 11), (1, 8, 8, 128, 8, 0),
                                   (3, 300, 2, 256, 1, 299), (2, 20, 5, 8, 7, 13)])
def test_append_bit_exact(combo, shape):
    cache_dt, new_dt, seq_major, new_hm = combo
    b, s, h, d, length, pos = shape
    x = make_cache_inputs(b, s, h, d, length, cache_dtype=cache_dt, new_dtype=new_dt,
                          seed=b * 1000 + s + d)
    if new_dt == torch.float32:
        # rounding edge cases in the first row of new keys: exact ties, a
        # carry past the largest bf16, infinities, a NaN, a subnormal
        flat = x["new_k"].view(-1)
        specials = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 65792.0, 3.4e38,
                                 float("inf"), -float("inf"), float("nan"), 2.0 ** -130])
        flat[:min(d, specials.numel())] = specials[:d]
    kc = to_layout(x["k_cache"], not seq_major).cuda()
    vc = to_layout(x["v_cache"], not seq_major).cuda()
    nk = to_layout(x["new_k"], new_hm).cuda()
    nv = to_layout(x["new_v"], new_hm).cuda()
    n = mgq.kv_append(kc, vc, nk, nv, pos, seq_major=seq_major, new_head_major=new_hm)
    torch.cuda.synchronize()
    want_k, want_v, want_n = okv.kv_update(bits_of(x["k_cache"]), bits_of(x["v_cache"]),
                                           bits_of(x["new_k"]), bits_of(x["new_v"]), pos)
    assert n == want_n
    assert_same_bits(bits_of(from_layout(kc.cpu(), not seq_major)), want_k, "key cache")
    assert_same_bits(bits_of(from_layout(vc.cpu(), not seq_major)), want_v, "value cache")


# Blocks large enough for the staged-runs kernel (a million new elements per
# tensor, runs of at least 1024 elements, cache and tokens in the same
# layout).  1030 tokens x 4 heads x 128: a (B, S, H, D) run is 128.75
# chunks of 4096 elements and a (B, H, S, D) run 32.19, so every run ends in
# a ragged chunk.  Ring positions: 4900 lands at slot 100 (no wrap, staged
# kernel); 5000 lands at slot 200 and wraps (generic kernel).
STAGED = [(cache_dt, new_dt, seq_major)
          for cache_dt in (torch.bfloat16, torch.float32)
          for new_dt in (torch.float32, torch.bfloat16)
          for seq_major in (True, False)]


@pytest.mark.parametrize("combo", STAGED, ids=[
    f"{str(c[0])[6:]}-new_{str(c[1])[6:]}-{'seq' if c[2] else 'head'}" for c in STAGED])
@pytest.mark.parametrize("where", [("linear", 100), ("ring", 4900), ("ring", 5000)])
def test_append_large_blocks_bit_exact(combo, where):
    cache_dt, new_dt, seq_major = combo
    mode, pos = where
    b, s, h, d, length = 2, 1200, 4, 128, 1030
    x = make_cache_inputs(b, s, h, d, length, cache_dtype=cache_dt, new_dtype=new_dt,
                          seed=7 + pos + d)
    kc = to_layout(x["k_cache"], not seq_major).cuda()
    vc = to_layout(x["v_cache"], not seq_major).cuda()
    nk = to_layout(x["new_k"], not seq_major).cuda()
    nv = to_layout(x["new_v"], not seq_major).cuda()
    ring = mode == "ring"
    n = mgq.kv_append(kc, vc, nk, nv, pos, seq_major=seq_major, new_head_major=not seq_major,
                      ring=ring)
    torch.cuda.synchronize()
    update = okv.ring_update if ring else okv.kv_update
    want_k, want_v, want_n = update(bits_of(x["k_cache"]), bits_of(x["v_cache"]),
                                    bits_of(x["new_k"]), bits_of(x["new_v"]), pos)
    assert n == want_n
    assert_same_bits(bits_of(from_layout(kc.cpu(), not seq_major)), want_k, "key cache")
    assert_same_bits(bits_of(from_layout(vc.cpu(), not seq_major)), want_v, "value cache")
    assert mgq.status() == 0


def test_append_page_examples():
    # The three worked examples printed on "KV Cache Update at a Position"
    # ("Examples": fp32 caches (B, S, H, D), fp32 new vectors), through the
    # append kernel.  Its head_dim is a multiple of 8, so each example's
    # vectors are zero-padded to 8 columns: the padded result must be the
    # page's output, padded the same way.
    import json

    from .kv_cache_pins import PAGE_EXAMPLES

    def pad8(a):
        a = np.asarray(a, dtype=np.float32)
        out = np.zeros(a.shape[:-1] + (8,), np.float32)
        out[..., :a.shape[-1]] = a
        return torch.from_numpy(out)

    with open(PAGE_EXAMPLES) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        kc, vc = pad8(c["key_cache"]).cuda(), pad8(c["value_cache"]).cuda()
        n = mgq.kv_append(kc, vc, pad8(c["new_keys"]).cuda(), pad8(c["new_values"]).cuda(),
                          c["position"])
        torch.cuda.synchronize()
        assert n == c["expected_length"], c["name"]
        assert torch.equal(kc.cpu(), pad8(c["expected_key_cache"])), c["name"]
        assert torch.equal(vc.cpu(), pad8(c["expected_value_cache"])), c["name"]


def test_append_edges():
    x = make_cache_inputs(2, 16, 2, 64, 16, seed=9)
    kc, vc = x["k_cache"].cuda(), x["v_cache"].cuda()
    before = kc.clone()
    empty = torch.empty(2, 0, 2, 64, device="cuda")
    assert mgq.kv_append(kc, vc, empty, empty, 16) == 16     # nothing to write at the end
    assert mgq.kv_append(kc, vc, empty, empty, 0) == 0
    torch.cuda.synchronize()
    assert torch.equal(kc, before)
    # a block filling the whole cache
    assert mgq.kv_append(kc, vc, x["new_k"].cuda(), x["new_v"].cuda(), 0) == 16
    torch.cuda.synchronize()
    assert torch.equal(kc.cpu(), x["new_k"].to(torch.bfloat16))


def test_append_rejects_blocks_that_do_not_fit():
    x = make_cache_inputs(1, 8, 1, 64, 3, seed=2)
    kc, vc = x["k_cache"].cuda(), x["v_cache"].cuda()
    nk, nv = x["new_k"].cuda(), x["new_v"].cuda()
    before = kc.clone()
    for pos in (-1, 6, 100):
        with pytest.raises(_lib.GqaAttnError) as e:
            mgq.kv_append(kc, vc, nk, nv, pos)
        assert e.value.code == -12
    flat = kc.view(-1)
    with pytest.raises(_lib.GqaAttnError) as e:    # new keys inside the key cache
        lib = _lib.load()
        rc = lib.gqa_attn_kv_append(kc.data_ptr(), vc.data_ptr(), flat.data_ptr() + 256,
                                    nv.data_ptr(), 1, 8, 1, 64, 0, 3, 0x4, None, None)
        _lib.check(rc, "gqa_attn_kv_append")
    assert e.value.code == -11
    torch.cuda.synchronize()
    assert torch.equal(kc, before)


DECODE_STEPS = [
    # (batch, slots, position, count, hq, hkv, d, causal, window, softcap, seq_major, new dtype)
    (4, 1500, 1000, 1, 32, 8, 128, True, None, None, True, torch.float32),
    (2, 9000, 8000, 4, 64, 4, 128, True, 4096, 30.0, True, torch.float32),
    (2, 700, 500, 40, 8, 2, 128, True, None, None, True, torch.bfloat16),   # tcgen05 path
    (1, 300, 0, 200, 4, 4, 64, True, 64, 20.0, False, torch.float32),      # from empty
    (3, 520, 77, 3, 12, 4, 96, False, None, None, False, torch.bfloat16),
    (2, 4100, 4000, 2, 16, 16, 72, True, 1000, None, True, torch.float32),
    (2, 600, 500, 20, 8, 2, 256, True, None, None, True, torch.float32),   # 2 row blocks write
    (1, 1100, 1000, 30, 4, 1, 256, True, 700, 25.0, False, torch.bfloat16),  # tokens span 2 tiles
]


@pytest.mark.parametrize("step", DECODE_STEPS, ids=[str(s[:10]) + ("seq" if s[10] else "head")
                                                    for s in DECODE_STEPS])
def test_decode_append_matches_oracle(step):
    b, s, pos, length, hq, hkv, d, causal, window, cap, seq_major, new_dt = step
    x = make_cache_inputs(b, s, hkv, d, length, new_dtype=new_dt, seed=s + pos,
                          num_q_heads=hq)
    kc = to_layout(x["k_cache"], not seq_major).cuda()
    vc = to_layout(x["v_cache"], not seq_major).cuda()
    q = x["q"].cuda()
    out = mgq.decode_append(q, kc, vc, x["new_k"].cuda(), x["new_v"].cuda(), pos,
                            seq_major=seq_major, causal=causal, window=window, softcap=cap)
    torch.cuda.synchronize()
    # oracle: update in the page's layout, then attend over the filled slots
    want_k, want_v, n = okv.kv_update(bits_of(x["k_cache"]), bits_of(x["v_cache"]),
                                      bits_of(x["new_k"]), bits_of(x["new_v"]), pos)
    assert n == pos + length
    assert_same_bits(bits_of(from_layout(kc.cpu(), not seq_major)), want_k, "key cache")
    assert_same_bits(bits_of(from_layout(vc.cpu(), not seq_major)), want_v, "value cache")
    k_used = bf16_from_bits(want_k[:, :n]).transpose(1, 2).contiguous()
    v_used = bf16_from_bits(want_v[:, :n]).transpose(1, 2).contiguous()
    want = oracle.attention(x["q"], k_used, v_used, causal=causal, window=window, softcap=cap)
    assert_close(out, want, f"decode_append {step[:10]}")
    # the same result, bit for bit, as attention on a contiguous copy
    ref = mgq.attention(q, k_used.cuda(), v_used.cuda(), causal=causal, window=window,
                        softcap=cap)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)


def test_decode_append_bench_workload_sampled():
    """The cache step the benchmark times, at full size, on sampled rows."""
    st = CACHE_STEPS["gqa_decode_append"]
    dev = torch.device("cuda")
    x = make_cache_inputs(st.batch, st.slots, st.num_kv_heads, st.head_dim, st.count,
                          seed=st.seed, num_q_heads=st.num_q_heads, device=dev)
    out = mgq.decode_append(x["q"], x["k_cache"], x["v_cache"], x["new_k"], x["new_v"],
                            st.position, seq_major=True, causal=st.causal, window=st.window,
                            softcap=st.softcap)
    torch.cuda.synchronize()
    n = st.kv_len
    k_used = x["k_cache"][:, :n].transpose(1, 2).contiguous().cpu()
    v_used = x["v_cache"][:, :n].transpose(1, 2).contiguous().cpu()
    # the appended slot holds the rounded new token
    want_slot = okv.f32_to_bf16_bits(x["new_k"].cpu().numpy()[:, 0])
    assert np.array_equal(bits_of(k_used[:, :, st.position]), want_slot)
    rng = np.random.default_rng(5)
    total = st.batch * st.num_q_heads * st.count
    rows = np.unique(np.concatenate([rng.choice(total, 96, replace=False), [0, total - 1]]))
    want = oracle.attention_rows(x["q"].cpu(), k_used, v_used, causal=st.causal,
                                 window=st.window, softcap=st.softcap, rows=rows)
    assert_close(out.reshape(-1, st.head_dim)[torch.as_tensor(rows)], want, st.name)


def test_fused_append_with_one_tile_per_split():
    """Every 64-key tile its own CTA: new tokens that straddle a tile edge
    are written by two CTAs, each before its own loads (decode kernel,
    head_dim 256, two row blocks)."""
    step = (1, 1100, 1000, 30, 4, 1, 256, True, None, None, True, torch.float32)
    mgq.set_override("tiles_per_split", 1)
    try:
        test_decode_append_matches_oracle(step)
    finally:
        mgq.set_override("tiles_per_split", 0)
