"""CUDA graph capture of the library's calls: a captured prefill (segmented plan, whose chunk kernel is
launched with programmatic stream serialization after the segment-state pass), varlen prefill (device-side
plan kernel), backward pass (three sweeps forked onto side streams and joined back through events) and
decode step (state updated in place) replay to the same bits as the eager calls, and read their input
buffers live at each replay.
"""

import pytest
import torch

from linear_attention_hybrid_b200 import (binding, la_decode_step, la_get_device_error, la_prefill,
                                          la_prefill_backward, la_prefill_varlen)
from linear_attention_hybrid_b200 import inputs as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def _capture(fn):
    """Run fn once on a side stream (first-use setup outside the capture), then capture it."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_prefill_graph_replay():
    B, N, H, D = 2, 3000, 8, 128   # 16 (sequence, head) pairs: a segmented plan (fp16 o: the corrected split)
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=3))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=4).to(DEV)
    ws = torch.empty(max(1, binding.la_prefill_workspace_size(B, N, H, D, out_dtype=torch.float16)),
                     dtype=torch.uint8, device=DEV)
    o = torch.empty(q.shape, dtype=torch.float16, device=DEV)
    sN = torch.empty_like(s0)
    run = lambda: la_prefill(q, k, v, initial_state=s0, final_state=sN, o=o, workspace=ws, out_dtype=torch.float16)
    g = _capture(run)
    o.zero_()
    sN.zero_()
    g.replay()
    torch.cuda.synchronize()
    o_eager, s_eager = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert torch.equal(o, o_eager) and torch.equal(sN, s_eager)
    # new inputs in the same buffers: the replay reads them
    q2, k2, v2 = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=9))
    q.copy_(q2), k.copy_(k2), v.copy_(v2)
    g.replay()
    torch.cuda.synchronize()
    o2, s2 = la_prefill(q2, k2, v2, initial_state=s0, return_final_state=True, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(sN, s2)


def test_varlen_graph_replay():
    lens = [700, 0, 5000, 129]
    cu = torch.tensor(W.cu_seqlens_of(lens), dtype=torch.int32, device=DEV)
    T, H, D = sum(lens), 8, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((T,), H, D, seed=5))
    ws = torch.empty(max(1, binding.la_prefill_varlen_workspace_size(T, len(lens), H, D)), dtype=torch.uint8,
                     device=DEV)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=DEV)
    sN = torch.empty((len(lens), H, D, D), dtype=torch.float32, device=DEV)
    g = _capture(lambda: la_prefill_varlen(q, k, v, cu, final_state=sN, o=o, workspace=ws))
    o.zero_()
    sN.zero_()
    g.replay()
    torch.cuda.synchronize()
    o_eager, s_eager = la_prefill_varlen(q, k, v, cu, return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(o, o_eager) and torch.equal(sN, s_eager)


def test_backward_graph_replay():
    B, N, H, D = 2, 2048, 8, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=6))
    g_out = W.make_grad_out((B, N), H, D, seed=7).to(DEV)
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=8).to(DEV)
    dsn = W.make_state((B,), H, D, D, std=0.1, seed=10).to(DEV)
    ws = torch.empty(max(1, binding.la_prefill_backward_workspace_size(B, N, H, D)), dtype=torch.uint8, device=DEV)
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
    ds0 = torch.empty_like(s0)
    run = lambda: la_prefill_backward(q, k, v, g_out, initial_state=s0, d_final_state=dsn, d_initial_state=ds0,
                                      dq=dq, dk=dk, dv=dv, workspace=ws)
    graph = _capture(run)
    for t in (dq, dk, dv, ds0):
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    want = la_prefill_backward(q, k, v, g_out, initial_state=s0, d_final_state=dsn, return_d_initial_state=True)
    torch.cuda.synchronize()
    for name, a, b in zip(("dq", "dk", "dv", "d_initial_state"), (dq, dk, dv, ds0), want):
        assert torch.equal(a, b), name


def test_decode_graph_replay():
    B, H, D, steps = 64, 16, 128, 5
    s_init = W.make_state((B,), H, D, D, std=0.1, seed=11).to(DEV)
    q, k, v = (x.to(DEV) for x in W.make_qkv((B,), H, D, seed=12))
    state = s_init.clone()
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=DEV)
    g = _capture(lambda: la_decode_step(q, k, v, state, o=o))
    state.copy_(s_init)
    for _ in range(steps):
        g.replay()
    torch.cuda.synchronize()
    ref = s_init.clone()
    for _ in range(steps):
        o_ref = la_decode_step(q, k, v, ref)
    torch.cuda.synchronize()
    assert torch.equal(state, ref) and torch.equal(o, o_ref)
