"""The C-ABI library: it loads, exports every declared symbol, and rejects
bad arguments before touching a device (CPU); error and status behaviour on
the GPU."""
import ctypes
import os
import re

import pytest
import torch

import masked_grouped_query_b200 as mgq
from masked_grouped_query_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gqa_attn.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gqa_attn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), f"{n} declared in gqa_attn.h but not exported"
    assert sorted(_lib.EXPORTS) == names


def test_version_and_error_strings(lib):
    assert lib.gqa_attn_version() >= 100
    for code in range(-12, 1):
        assert lib.gqa_attn_error_string(code)
    assert _lib.error_string(-4).startswith("num_q_heads")


def _fwd(lib, q=16, k=16, v=16, o=4096, dims=(1, 4, 4, 4, 2, 64, 1, 0), cap=0.0):
    P = ctypes.c_void_p
    return lib.gqa_attn_fwd(P(q), P(k), P(v), P(o), *dims, cap, None)


@pytest.mark.parametrize("dims,cap,code", [
    ((1, 4, 4, 3, 2, 64, 1, 0), 0.0, -4),      # 3 q heads over 2 kv heads
    ((1, 4, 4, 4, 2, 60, 1, 0), 0.0, -5),      # head_dim not a multiple of 8
    ((1, 4, 4, 4, 2, 264, 1, 0), 0.0, -5),     # head_dim > 256
    ((1, 4, 4, 4, 2, 0, 1, 0), 0.0, -5),
    ((-1, 4, 4, 4, 2, 64, 1, 0), 0.0, -3),     # negative batch
    ((1, 4, 4, 0, 2, 64, 1, 0), 0.0, -3),      # zero heads
    ((1, 4, 4, 4, 2, 64, 1, 0), -1.0, -6),     # negative softcap
    ((1, 4, 4, 4, 2, 64, 1, 0), float("nan"), -6),
    ((1, 4, 4, 4, 2, 64, 1, 0), float("inf"), -6),
])
def test_rejects_bad_sizes_without_a_device(lib, dims, cap, code):
    assert _fwd(lib, dims=dims, cap=cap) == code


def test_rejects_bad_pointers_without_a_device(lib):
    assert _fwd(lib, q=0) == -1                      # null q with elements
    assert _fwd(lib, k=0) == -1
    assert _fwd(lib, q=24) == -2                     # misaligned
    assert _fwd(lib, q=0x10000, o=0x10000 + 64) == -11   # o overlaps q
    big = (1, 1 << 20, 4, 1 << 12, 1, 256, 1, 0)     # rows per kv head >= 2^31
    assert _fwd(lib, dims=big) == -10


def _append(lib, kc=0x1000, vc=0x100000, nk=0x200000, nv=0x300000, b=1, s=8, h=2, d=64,
            pos=0, n=1, flags=0):
    P = ctypes.c_void_p
    return lib.gqa_attn_kv_append(P(kc), P(vc), P(nk), P(nv), b, s, h, d, pos, n, flags,
                                  None, None)


def test_append_rejects_bad_arguments_without_a_device(lib):
    assert _append(lib, pos=-1) == -12
    assert _append(lib, pos=8) == -12            # 8 + 1 > 8 slots
    assert _append(lib, pos=5, n=4) == -12
    assert _append(lib, flags=0x20) == -12       # unknown flag
    assert _append(lib, flags=0x10, pos=100) == -7   # ring: any position (then: no device)
    assert _append(lib, flags=0x10, n=9) == -12      # ring: block larger than the ring
    assert _append(lib, d=60) == -5
    assert _append(lib, h=0) == -3
    assert _append(lib, kc=0) == -1
    assert _append(lib, nk=0x200008) == -2
    assert _append(lib, vc=0x1000 + 64) == -11   # caches overlap
    assert _append(lib, nk=0x1000 + 512) == -11  # new keys inside the key cache
    assert _append(lib, n=0, kc=0) == 0          # nothing to write: no device needed
    length = ctypes.c_int(-1)
    P = ctypes.c_void_p
    assert lib.gqa_attn_kv_append(P(0), P(0), P(0), P(0), 1, 8, 2, 64, 3, 0, 0,
                                  ctypes.byref(length), None) == 0
    assert length.value == 3
    # the decode step takes bf16 caches only, and checks the block fits
    q = o = None
    assert lib.gqa_attn_decode_append(P(0x10000), P(0x20000), P(0x80000), P(0x100000),
                                      P(0x110000), P(0x120000), 1, 1, 7, 8, 4, 2, 64, 0x2,
                                      1, 0, 0.0, None) == -12
    assert lib.gqa_attn_decode_append(P(0x10000), P(0x20000), P(0x80000), P(0x100000),
                                      P(0x110000), P(0x120000), 1, 2, 7, 8, 4, 2, 64, 0,
                                      1, 0, 0.0, None) == -12
    assert lib.gqa_attn_decode_append(P(0x20000), P(0x20000), P(0x80000), P(0x100000),
                                      P(0x110000), P(0x120000), 1, 1, 7, 8, 4, 2, 64, 0,
                                      1, 0, 0.0, None) == -11   # q inside the key cache
    del q, o


def _ring(lib, kv_len=5000, slots=4096, q_len=1, window=4096, flags=0, d=64):
    P = ctypes.c_void_p
    return lib.gqa_attn_fwd_ring(P(0x10000), P(0x100000), P(0x800000), P(0x2000000), 1, q_len,
                                 kv_len, slots, 4, 2, d, flags, 1, window, 0.0, None)


def test_ring_rejects_bad_arguments_without_a_device(lib):
    assert _ring(lib, slots=4000) == -12                  # not whole 64-key tiles
    assert _ring(lib, slots=0) == -12
    assert _ring(lib, q_len=2) == -12                     # needs window + 1 = 4097 slots
    assert _ring(lib, window=0) == -12                    # no window: all 5000 keys visible
    assert _ring(lib, window=0, kv_len=4096) == -7        # they fit: then no device
    assert _ring(lib, flags=0x2) == -12                   # only the layout flag is accepted
    assert _ring(lib) == -7
    assert _ring(lib, flags=0x1) == -7


def test_override_keys(lib):
    # Keys 1-5 are knobs (host state only, no device needed); others are rejected.
    for key in (1, 2, 3, 4, 5):
        assert lib.gqa_attn_set_override(key, 0) == 0
    assert lib.gqa_attn_set_override(4, -1) == 0
    assert lib.gqa_attn_set_override(4, 0) == 0
    assert lib.gqa_attn_set_override(5, 1) == 0
    assert lib.gqa_attn_set_override(5, 0) == 0
    assert lib.gqa_attn_set_override(6, 0) == -12  # GQA_ATTN_ERR_ARG
    assert lib.gqa_attn_set_override(0, 0) == -12
    with pytest.raises(KeyError):
        mgq.set_override("no_such_knob", 1)


def test_no_device_means_device_error(lib):
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    assert _fwd(lib) == -7
    assert lib.gqa_attn_selftest_bounded_wait(100, None) == -7
    assert _append(lib) == -7


def test_empty_problem_is_a_no_op(lib):
    # batch 0 / q_len 0: nothing to compute, nothing dereferenced.
    for dims in [(0, 4, 4, 4, 2, 64, 1, 0), (1, 0, 4, 4, 2, 64, 1, 0)]:
        rc = _fwd(lib, q=0, k=16, v=16, o=0, dims=dims)
        assert rc in (0, -7)


@pytest.mark.gpu
def test_bad_arguments_raise_from_python():
    q = torch.zeros(1, 3, 4, 64, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.GqaAttnError) as e:
        mgq.attention(q, k, k)
    assert e.value.code == -4
    with pytest.raises(TypeError):
        mgq.attention(q.float(), k, k)


@pytest.mark.gpu
def test_status_word_and_bounded_wait_selftest():
    mgq.clear_status()
    torch.cuda.synchronize()
    assert mgq.status() == 0
    mgq.selftest_bounded_wait(2000)
    torch.cuda.synchronize()
    assert mgq.status() & 0x20
    mgq.clear_status()
    assert mgq.status() == 0
    # The context is still usable afterwards.
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


@pytest.mark.gpu
def test_output_guard_regions_untouched():
    w = mgq.Workload("g", 2, 5, 70, 8, 2, 64, True, 9, 20.0, 3)
    q, k, v = mgq.make_inputs(w)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    n = q.numel()
    buf = torch.full((n + 2 * 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[4096:4096 + n].view(q.shape)
    mgq.attention(q, k, v, causal=True, window=9, softcap=20.0, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:4096] == 7.0) and torch.all(buf[4096 + n:] == 7.0)
    assert torch.isfinite(out.float()).all()
