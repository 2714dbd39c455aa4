"""la_prefill_noalloc: the prefill entry point for callers that cannot allocate
device scratch (for example code running under a host framework that owns all
device memory, or a latency path that cannot afford cudaMalloc's device-wide
synchronisation). It must give the same results as la_prefill with a caller
workspace, and the library-owned scratch it reuses must not carry state from
one call into the next.

Kept in a file that pytest collects last: it is the newest addition, so a run
that stops at the first failure has already run everything else.
"""

import pytest
import torch

from linear_attention_hybrid_b200 import la_get_device_error, la_prefill, la_prefill_noalloc
from linear_attention_hybrid_b200 import binding
from linear_attention_hybrid_b200 import inputs as W
from tests.parity_util import check, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # B*H small and N long: the segment split runs, so the static scratch holds segment states
    B, N, H, D = 1, 3000, 2, 128
    assert binding.la_prefill_workspace_size(B, N, H, D) > 0
    for call, seed in enumerate((21, 22)):     # two calls in a row, different inputs
        q, k, v = (x.to("cuda") for x in W.make_qkv((B, N), H, D, seed=seed))
        s0 = W.make_state((B,), H, D, D, seed=seed + 100).to("cuda")
        o_ref, s_ref = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=torch.float16)
        o, s = la_prefill_noalloc(q, k, v, initial_state=s0, return_final_state=True, out_dtype=torch.float16)
        torch.cuda.synchronize()
        check(to64(o), to64(o_ref), torch.bfloat16, f"call {call} o")
        check(to64(s), to64(s_ref), torch.bfloat16, f"call {call} final state")


def test_noalloc_rejects_calls_beyond_its_scratch(monkeypatch):
    # default planning keeps a uniform batch's scratch well inside the fixed array, so force
    # 128-token segments (LA_SEG_LEN): 8 heads x 512 segment states need far more than 32 MiB
    monkeypatch.setenv("LA_SEG_LEN", "128")
    B, N, H, D = 1, 65536, 8, 128
    assert binding.la_prefill_workspace_size(B, N, H, D) > 32 << 20
    L = binding.lib()
    fake = 0x10000000   # never dereferenced: the size check comes first
    st = L.la_prefill_noalloc(fake, fake * 2, fake * 3, fake * 4, B, N, H, D, 0, None, None, None, None)
    assert st == binding.LA_ERR_WORKSPACE
    assert "scratch" in binding.la_last_error()
