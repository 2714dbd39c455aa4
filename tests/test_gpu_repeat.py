"""Repeated and concurrent calls: results are deterministic across back-to-back calls and unchanged when two
prefills run on two streams at once, and no call stalls. The stall guard proper is on the device: every wait in
the kernels is bounded and records LA_ERR_DEVICE_TIMEOUT when it runs out, which the fixture reads after each
test. The host clock only catches a gross stall (ten calls normally take about 2 ms; the limit is 10 s, far
above what a busy or preempted host adds)."""

import time

import pytest
import torch

from linear_attention_hybrid_b200 import binding, la_get_device_error, la_prefill, la_prefill_backward
from linear_attention_hybrid_b200 import inputs as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def test_backward_repeats_bit_for_bit_without_stalls():
    """8 (sequence, head) pairs: the three sweeps each run a segmented plan (state pass, then the chunk
    kernel through programmatic dependent launch) on three streams at once."""
    B, N, H, D = 2, 8192, 4, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=21))
    g = W.make_grad_out((B, N), H, D, seed=22).to(DEV)
    ws = torch.empty(binding.la_prefill_backward_workspace_size(B, N, H, D), dtype=torch.uint8, device=DEV)
    dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
    la_prefill_backward(q, k, v, g, dq=dq, dk=dk, dv=dv, workspace=ws)
    torch.cuda.synchronize()
    ref = [t.clone() for t in (dq, dk, dv)]
    for _ in range(10):
        t0 = time.perf_counter()
        for _ in range(10):
            la_prefill_backward(q, k, v, g, dq=dq, dk=dk, dv=dv, workspace=ws)
        torch.cuda.synchronize()
        assert time.perf_counter() - t0 < 10.0, "ten backward calls took over ten seconds"
        for a, b in zip((dq, dk, dv), ref):
            assert torch.equal(a, b)


def test_two_prefills_on_two_streams_match_one_stream():
    B, N, H, D = 2, 4096, 16, 128   # 32 pairs: a segmented plan per call
    ins = [tuple(x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=s)) for s in (31, 32)]
    want = []
    for q, k, v in ins:
        o, s = la_prefill(q, k, v, return_final_state=True, out_dtype=torch.float16)
        want.append((o, s))
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in ins]
    wss = [torch.empty(binding.la_prefill_workspace_size(B, N, H, D, out_dtype=torch.float16), dtype=torch.uint8, device=DEV) for _ in ins]
    outs = [(torch.empty_like(w[0]), torch.empty_like(w[1])) for w in want]
    for _ in range(20):
        for st, (q, k, v), (o, s), ws in zip(streams, ins, outs, wss):
            st.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(st):
                la_prefill(q, k, v, o=o, final_state=s, workspace=ws, out_dtype=torch.float16)
        for st in streams:
            torch.cuda.current_stream().wait_stream(st)
        torch.cuda.synchronize()
        for (o, s), (wo, ws_) in zip(outs, want):
            assert torch.equal(o, wo) and torch.equal(s, ws_)
