"""GPU parity of the fused output norm + gate (la_prefill_norm_gate, la_prefill_varlen_norm_gate,
la_decode_steps_norm_gate) against the oracle: the operator's output followed by
y = w_h * o / sqrt(mean(o^2) + eps) * sigmoid(z) per (token, head), in fp64. The bound is the operator's,
against the RMS of the oracle's y (plus half a bf16 ulp of the value for a bf16 y)."""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_hybrid_b200 import (la_decode_steps_norm_gate, la_get_device_error, la_last_launch_count,
                                          la_norm_gate, la_prefill, la_prefill_norm_gate, la_prefill_varlen_norm_gate)
from linear_attention_hybrid_b200 import inputs as W
from tests.parity_util import check, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
EPS = 1e-6


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def _want(q, k, v, z, w, s0=None, cu=None, lam=None):
    H = q.shape[-2]
    return oracle.prefill_norm_gate(q, k, v, z, w, EPS, cu_seqlens=cu, lam=oracle.decay(H) if lam is None else lam,
                                    initial_state=s0, return_final_state=True)


@pytest.mark.parametrize("N", [1, 127, 129, 1000, 2177])
@pytest.mark.parametrize("out", [torch.float16, torch.float32, torch.bfloat16])
def test_prefill_norm_gate_ragged(N, out):
    B, H, D = 2, 3, 128
    q, k, v = W.make_qkv((B, N), H, D, seed=N)
    z, w = W.make_norm_gate((B, N), H, D, seed=N + 1)
    s0 = W.make_state((B,), H, D, D, seed=N + 2)
    y, sN = la_prefill_norm_gate(*(x.to(DEV) for x in (q, k, v, z, w)), eps=EPS, initial_state=s0.to(DEV),
                                 return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    want_y, want_s = _want(q, k, v, z, w, s0)
    check(to64(y), want_y, torch.bfloat16, "y", stored_bf16=out == torch.bfloat16)
    check(to64(sN), want_s, torch.bfloat16, "final state")


def test_prefill_norm_gate_workload_shape():
    """The prefill workload's shape (B=4, N=4096, H=16: two segments per sequence), fp16 y, every element."""
    B, N, H, D = 4, 4096, 16, 128
    q, k, v = W.make_qkv((B, N), H, D, seed=0)
    z, w = W.make_norm_gate((B, N), H, D, seed=1)
    y = la_prefill_norm_gate(*(x.to(DEV) for x in (q, k, v, z, w)), eps=EPS, out_dtype=torch.float16)
    torch.cuda.synchronize()
    check(to64(y), _want(q, k, v, z, w)[0], torch.bfloat16, "y")


def test_prefill_norm_gate_segmented_long():
    B, N, H, D = 1, 6000, 2, 128
    q, k, v = W.make_qkv((B, N), H, D, seed=5)
    z, w = W.make_norm_gate((B, N), H, D, seed=6)
    y, sN = la_prefill_norm_gate(*(x.to(DEV) for x in (q, k, v, z, w)), eps=EPS, return_final_state=True,
                                 out_dtype=torch.float32)
    torch.cuda.synchronize()
    want_y, want_s = _want(q, k, v, z, w)
    check(to64(y), want_y, torch.bfloat16, "y")
    check(to64(sN), want_s, torch.bfloat16, "final state")


def test_prefill_norm_gate_final_state_equals_plain_prefill():
    """The epilogue changes only the output: the final state is bit for bit the plain prefill's."""
    B, N, H, D = 2, 1500, 4, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=7))
    z, w = (x.to(DEV) for x in W.make_norm_gate((B, N), H, D, seed=8))
    _, s_plain = la_prefill(q, k, v, return_final_state=True)
    _, s_gated = la_prefill_norm_gate(q, k, v, z, w, eps=EPS, return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(s_plain, s_gated)


def test_varlen_norm_gate_with_guard_bands():
    lens = [0, 1, 127, 129, 700, 3000, 5]
    H, D, pad = 2, 128, 64
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v = W.make_qkv((T,), H, D, seed=12)
    z, w = W.make_norm_gate((T,), H, D, seed=13)
    big = torch.full((T + 2 * pad, H, D), float("nan"), dtype=torch.float16, device=DEV)
    y = big[pad:pad + T]
    cu_d = torch.tensor(cu, dtype=torch.int32, device=DEV)
    la_prefill_varlen_norm_gate(*(x.to(DEV) for x in (q, k, v, z, w)), cu_d, eps=EPS, o=y)
    torch.cuda.synchronize()
    assert torch.isnan(big[:pad].float()).all() and torch.isnan(big[pad + T:].float()).all(), "wrote outside o"
    check(to64(y), _want(q, k, v, z, w, cu=cu)[0], torch.bfloat16, "y")


@pytest.mark.parametrize("dtype, out, D", [(torch.bfloat16, torch.float16, 128), (torch.bfloat16, torch.bfloat16, 128),
                                           (torch.bfloat16, torch.float32, 64), (torch.float32, torch.float32, 128)])
@pytest.mark.parametrize("K", [1, 3, 16])
def test_decode_norm_gate(dtype, out, D, K):
    B, H = 6, 4
    q, k, v = W.make_qkv((B, K), H, D, dtype=dtype, seed=K + D)
    z, w = W.make_norm_gate((B, K), H, D, dtype=dtype, seed=K + D + 1)
    s0 = W.make_state((B,), H, D, D, seed=3)
    st = s0.clone().to(DEV)
    y = la_decode_steps_norm_gate(*(x.to(DEV) for x in (q, k, v, z, w)), st, eps=EPS, out_dtype=out)
    torch.cuda.synchronize()
    want_y, want_s = _want(q, k, v, z, w, s0)
    check(to64(y), want_y, dtype, "y", stored_bf16=out == torch.bfloat16)
    check(to64(st), want_s, dtype, "state")


def test_decode_norm_gate_equals_prefill_norm_gate():
    """K decode steps with the epilogue give the prefill-with-epilogue output of the same K tokens."""
    B, K, H, D = 3, 24, 4, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, K), H, D, seed=30))
    z, w = (x.to(DEV) for x in W.make_norm_gate((B, K), H, D, seed=31))
    st = torch.zeros((B, H, D, D), dtype=torch.float32, device=DEV)
    yd = la_decode_steps_norm_gate(q, k, v, z, w, st, eps=EPS, out_dtype=torch.float32)
    yp = la_prefill_norm_gate(q, k, v, z, w, eps=EPS, out_dtype=torch.float32)
    torch.cuda.synchronize()
    check(to64(yd), to64(yp), torch.bfloat16, "decode vs prefill")


@pytest.mark.parametrize("dtype, out, D", [(torch.float32, torch.float32, 128), (torch.float32, torch.float32, 64),
                                           (torch.bfloat16, torch.bfloat16, 64), (torch.bfloat16, torch.float16, 64)])
def test_prefill_norm_gate_fp32_and_d64_paths(dtype, out, D):
    B, N, H = 2, 300, 3
    q, k, v = W.make_qkv((B, N), H, D, dtype=dtype, seed=D)
    z, w = W.make_norm_gate((B, N), H, D, dtype=dtype, seed=D + 1)
    s0 = W.make_state((B,), H, D, D, seed=D + 2)
    y, sN = la_prefill_norm_gate(*(x.to(DEV) for x in (q, k, v, z, w)), eps=EPS, initial_state=s0.to(DEV),
                                 return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    want_y, want_s = _want(q, k, v, z, w, s0)
    check(to64(y), want_y, dtype, "y", stored_bf16=out == torch.bfloat16)
    check(to64(sN), want_s, dtype, "final state")


@pytest.mark.parametrize("odt, gdt, D", [(torch.float16, torch.bfloat16, 128), (torch.bfloat16, torch.bfloat16, 128),
                                         (torch.float32, torch.bfloat16, 64), (torch.float32, torch.float32, 128)])
@pytest.mark.parametrize("in_place", [False, True])
def test_norm_gate_alone(odt, gdt, D, in_place):
    """The streaming pass on its own, against the oracle applied to the same (rounded) o."""
    T, H = 1000, 5
    o = (torch.randn((T, H, D), generator=torch.Generator().manual_seed(D)) * 0.3).to(odt)
    z, w = W.make_norm_gate((T,), H, D, dtype=gdt, seed=4)
    od, zd, wd = o.to(DEV), z.to(DEV), w.to(DEV)
    y = la_norm_gate(od, zd, wd, eps=EPS, y=od if in_place else None)
    torch.cuda.synchronize()
    assert la_last_launch_count() == 1
    want = oracle.norm_gate(o.double().numpy(), z.double().numpy(), w.double().numpy(), EPS)
    check(to64(y), want, torch.float32 if gdt == torch.float32 else torch.bfloat16, "y",
          stored_bf16=odt == torch.bfloat16)
    if in_place:
        assert y.data_ptr() == od.data_ptr()


def test_prefill_norm_gate_launches():
    B, N, H, D = 10, 300, 16, 128   # unsegmented: the chunk kernel, then the norm + gate pass
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=3))
    z, w = (x.to(DEV) for x in W.make_norm_gate((B, N), H, D, seed=4))
    la_prefill_norm_gate(q, k, v, z, w, eps=EPS)
    assert la_last_launch_count() == 2
