"""la_prefill_noalloc: the prefill entry point for callers that cannot allocate
device scratch (for example code running under a host framework that owns all
device memory, or a latency path that cannot afford cudaMalloc's device-wide
synchronisation). It runs the same kernels on the same plan as la_prefill with a
caller workspace, so its results must be the same bits; and the library-owned
scratch it reuses must not carry anything from one call into the next.

Kept in a file that pytest collects last: it is the newest addition, so a run
that stops at the first failure has already run everything else.
"""

import pytest
import torch

from linear_attention_hybrid_b200 import la_get_device_error, la_prefill, la_prefill_noalloc
from linear_attention_hybrid_b200 import binding
from linear_attention_hybrid_b200 import inputs as W

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0


def _both(B, N, H, D, seed, dtype=torch.bfloat16, out_dtype=torch.float16):
    """One la_prefill_noalloc call and the same call through la_prefill with a caller workspace."""
    q, k, v = (x.to("cuda") for x in W.make_qkv((B, N), H, D, dtype=dtype, seed=seed))
    s0 = W.make_state((B,), H, D, D, seed=seed + 100).to("cuda")
    ws_bytes = binding.la_prefill_workspace_size(B, N, H, D, dtype, out_dtype)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    o_ref, s_ref = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out_dtype, workspace=ws)
    o, s = la_prefill_noalloc(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out_dtype)
    torch.cuda.synchronize()
    return ws_bytes, (o, s), (o_ref, s_ref)


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # Three calls in a row on one stream, each compared bit for bit with la_prefill:
    #   1. many (sequence, head) states in the scratch (a long sequence over few heads: many segments),
    #   2. a different, smaller shape whose plan covers only part of what call 1 left in the scratch,
    #   3. fp32 inputs (the CUDA-core path), which need no scratch at all.
    calls = [(1, 20000, 2, 128, 21, torch.bfloat16), (2, 3000, 4, 64, 22, torch.bfloat16),
             (1, 700, 2, 64, 23, torch.float32)]
    sizes = []
    for i, (B, N, H, D, seed, dtype) in enumerate(calls):
        out_dtype = torch.float16 if dtype == torch.bfloat16 else torch.float32
        ws_bytes, (o, s), (o_ref, s_ref) = _both(B, N, H, D, seed, dtype, out_dtype)
        sizes.append(ws_bytes)
        assert torch.equal(o, o_ref), f"call {i}: o differs from la_prefill's"
        assert torch.equal(s, s_ref), f"call {i}: final state differs from la_prefill's"
    assert sizes[0] > sizes[1] > 0 and sizes[2] == 0, sizes
