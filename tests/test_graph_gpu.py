"""The attention call inside a CUDA graph (GPU).

After one call on a stream (which sizes that stream's split workspace), a
call enqueues only kernels -- no allocation, no host synchronisation -- so a
serving loop can capture it once and replay it: the tensor maps and plan are
baked in at capture, and replays read whatever the captured buffers hold.
"""
import pytest
import torch

import masked_grouped_query_b200 as mgq
from masked_grouped_query_b200.inputs import Workload, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [
    Workload("decode", 4, 1, 3000, 32, 8, 128, True, None, None, 31),         # split-KV decode
    Workload("prefill", 1, 300, 900, 8, 2, 128, True, 256, 30.0, 32),         # tcgen05, key splits
    Workload("clustered", 8, 4, 5000, 64, 4, 128, True, 2048, 30.0, 33),      # 4-CTA cluster merge
])
def test_captured_call_replays_like_a_direct_call(w):
    if w.name == "clustered":  # the cluster merge also writes its partials to the workspace
        plan = mgq.describe(w.batch, w.q_len, w.kv_len, w.num_q_heads, w.num_kv_heads,
                            w.head_dim, w.causal, w.window, w.softcap)
        assert plan["cluster"] >= 2, plan
    q, k, v = (t.cuda() for t in make_inputs(w))
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mgq.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap, out=out)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        mgq.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap, out=out)
    for seed in (1, 2):
        q2, k2, v2 = make_inputs(w, seed=100 + seed)
        q.copy_(q2)
        k.copy_(k2)
        v.copy_(v2)
        g.replay()
        torch.cuda.synchronize()
        want = mgq.attention(q, k, v, causal=w.causal, window=w.window, softcap=w.softcap)
        torch.cuda.synchronize()
        assert torch.equal(out, want)
    assert mgq.status() & 0x1f == 0


def test_captured_call_survives_workspace_growth():
    # A graph captured with a small split call keeps valid workspace
    # pointers after a larger direct call on the same stream grows the
    # stream's workspace (the old buffers are retired, not freed).
    from oracle import oracle

    small = Workload("small", 1, 1, 4000, 8, 2, 128, True, None, None, 41)
    big = Workload("big", 16, 1, 60000, 32, 8, 128, True, None, None, 42)
    q, k, v = (t.cuda() for t in make_inputs(small))
    out = torch.empty_like(q)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        mgq.attention(q, k, v, causal=True, out=out)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        mgq.attention(q, k, v, causal=True, out=out)
    qb, kb, vb = (t.cuda() for t in make_inputs(big))
    plan_s = mgq.describe(1, 1, 4000, 8, 2, 128, True)
    plan_b = mgq.describe(16, 1, 60000, 32, 8, 128, True)
    assert plan_s["splits"] > 1 and plan_b["splits"] * plan_b["ctas"] > plan_s["splits"] * plan_s["ctas"]
    with torch.cuda.stream(s):
        ob = mgq.attention(qb, kb, vb, causal=True)   # grows the stream's workspace
    s.synchronize()
    q2, k2, v2 = make_inputs(small, seed=143)
    q.copy_(q2)
    k.copy_(k2)
    v.copy_(v2)
    with torch.cuda.stream(s):
        g.replay()
    s.synchronize()
    want = oracle.attention(q2, k2, v2, causal=True, window=None, softcap=None)
    got = out.float().cpu().numpy()
    assert abs(got - want).max() <= 2e-2 and ((abs(got - want) <= 2e-2 + 2e-2 * abs(want)).all())
    assert torch.isfinite(ob).all()
    del g
    assert mgq.status() & 0x1f == 0
