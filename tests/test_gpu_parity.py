"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases compare every output element and every final-state entry; the
specified full-size workloads compare sampled (sequence, head) slices, each
slice over its whole length, in the same launch configuration the benchmark
uses. Every test also checks that no kernel recorded a device-side status.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_hybrid_b200 import (la_decode_step, la_decode_steps, la_get_device_error, la_last_launch_count, la_prefill,
                                          la_prefill_varlen)
from linear_attention_hybrid_b200 import inputs as W
from tests.parity_util import check, oracle_heads, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
# the output type bench.py times: bf16 q, k, v in, fp16 o out (held to the bound with no allowance)
BENCH_OUT = torch.float16


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def _lam(H):
    return oracle.decay(H)


def _full_compare(q, k, v, s0, dtype, o, sN, lam=None, cu=None):
    """Oracle over every sequence and head; q etc. are [B, N, H, D] or [T, H, D] CUDA tensors."""
    H = q.shape[-2]
    lam = _lam(H) if lam is None else lam
    want_o, want_s = oracle.prefill_recurrent(q, k, v, cu_seqlens=cu, lam=lam,
                                              initial_state=None if s0 is None else s0.cpu(), return_final_state=True)
    check(to64(o), want_o, dtype, "o", stored_bf16=o.dtype == torch.bfloat16)
    if sN is not None:
        check(to64(sN).reshape(want_s.shape), want_s, dtype, "final state")


# --------------------------------------------------------------------------- the tiny fp32 workload
def test_tiny_fp32_workload():
    wl = W.workloads()["tiny_fp32"]
    q, k, v = (x.to(DEV) for x in W.make_qkv((wl.B, wl.N), wl.H, wl.D, dtype=wl.dtype, seed=wl.seed))
    o, sN = la_prefill(q, k, v, return_final_state=True)
    torch.cuda.synchronize()
    _full_compare(q, k, v, None, torch.float32, o, sN)


# --------------------------------------------------------------------------- bf16 tensor-core path, small sizes
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 256, 300, 1000, 2177])
@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("out", [torch.float16, torch.float32, torch.bfloat16])
def test_prefill_bf16_ragged(N, with_state, out):
    B, H, D = 2, 3, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=N))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=N + 1).to(DEV) if with_state else None
    o, sN = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    _full_compare(q, k, v, s0, torch.bfloat16, o, sN)


def test_prefill_bf16_unsegmented_many_heads():
    B, N, H, D = 10, 300, 16, 128   # B*H >= 148: one unit per (sequence, head), no workspace states
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=3))
    o, sN = la_prefill(q, k, v, return_final_state=True)
    torch.cuda.synchronize()
    assert la_last_launch_count() == 1   # uniform batch, no segment split: the chunk kernel alone
    _full_compare(q, k, v, None, torch.bfloat16, o, sN)


def test_prefill_segmented_launches():
    B, N, H, D = 1, 1000, 2, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=4))
    la_prefill(q, k, v, out_dtype=torch.float16)   # the corrected split (uniform batches need no plan kernel)
    assert la_last_launch_count() == 3   # chunk kernel, entry states, output correction
    la_prefill(q, k, v, out_dtype=torch.bfloat16)
    assert la_last_launch_count() == 2   # bf16 output: segment-state pass + chunk kernel


# 64 (sequence, head) pairs: two segments per sequence, whose output correction splits each entry state itself
# and forms the final states (N = 300 ends the second segment in a partial chunk)
@pytest.mark.parametrize("out", [torch.float16, torch.float32])
@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("N", [300, 1000, 2177])
def test_prefill_two_segments_corrected(N, with_state, out):
    B, H, D = 4, 16, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=N + 50))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=N + 51).to(DEV) if with_state else None
    o, sN = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    assert la_last_launch_count() == 2   # chunk kernel, output correction (the entry states need no grid)
    _full_compare(q, k, v, s0, torch.bfloat16, o, sN)


def test_prefill_two_segments_final_state_in_place():
    B, N, H, D = 4, 1000, 16, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=61))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=62).to(DEV)
    ref_o, ref_s = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=torch.float16)
    st = s0.clone()
    o, _ = la_prefill(q, k, v, initial_state=st, final_state=st, out_dtype=torch.float16)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o) and torch.equal(st, ref_s)


# fp32 inputs (CUDA cores) and bf16 with D = 64 (tensor cores, the D = 64 instances) around the 64-token chunk
@pytest.mark.parametrize("dtype, out, D", [(torch.float32, torch.float32, 128), (torch.float32, torch.float32, 64),
                                           (torch.bfloat16, torch.bfloat16, 64), (torch.bfloat16, torch.float32, 64),
                                           (torch.bfloat16, torch.float16, 64)])
@pytest.mark.parametrize("N", [1, 63, 64, 65, 300])
def test_prefill_fp32_and_d64_paths(dtype, out, D, N):
    B, H = 2, 3
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, dtype=dtype, seed=N + D))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=5).to(DEV)
    o, sN = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    _full_compare(q, k, v, s0, dtype, o, sN)


# --------------------------------------------------------------------------- D = 64, bf16: the chunk kernel's D = 64
# instance (one 64-column slab per operand, Q S on [S_hi | S_lo]) and the correction's, beside the zero-padded
# segment-state and entry-state kernels
# (segmented plans, states, ragged ends, every output type)
@pytest.mark.parametrize("B, N, H", [(1, 8192, 2), (2, 3000, 4), (3, 1337, 20), (10, 300, 16)])
@pytest.mark.parametrize("out", [torch.float16, torch.bfloat16, torch.float32])
def test_prefill_d64_tensor_core(B, N, H, out):
    D = 64
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=B * N + H))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=7).to(DEV)
    o, sN = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    assert la_last_launch_count() >= 1
    _full_compare(q, k, v, s0, torch.bfloat16, o, sN)


def test_prefill_d64_final_state_in_place():
    """final_state may alias initial_state; with D = 64 the states are read and written as 64 x 64."""
    B, N, H, D = 1, 5000, 4, 64
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=12))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=13).to(DEV)
    st = s0.clone()
    o, sN = la_prefill(q, k, v, initial_state=st, final_state=st)
    torch.cuda.synchronize()
    assert sN.data_ptr() == st.data_ptr()
    _full_compare(q, k, v, s0, torch.bfloat16, o, sN)


def test_varlen_d64_tensor_core():
    lens = [700, 0, 5000, 129, 2048]
    cu = W.cu_seqlens_of(lens)
    T, H, D = int(cu[-1]), 8, 64
    q, k, v = (x.to(DEV) for x in W.make_qkv((T,), H, D, seed=14))
    s0 = W.make_state((len(lens),), H, D, D, std=0.1, seed=15).to(DEV)
    o, sN = la_prefill_varlen(q, k, v, torch.tensor(cu, dtype=torch.int32, device=DEV), initial_state=s0,
                              return_final_state=True, out_dtype=torch.float16)
    torch.cuda.synchronize()
    _full_compare(q, k, v, s0, torch.bfloat16, o, sN, cu=cu)


def test_prefill_zero_length_passes_state_through():
    B, N, H, D = 2, 0, 3, 128
    q = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=DEV)
    s0 = W.make_state((B,), H, D, D, seed=6).to(DEV)
    o, sN = la_prefill(q, q.clone(), q.clone(), initial_state=s0, return_final_state=True)
    torch.cuda.synchronize()
    assert torch.equal(sN, s0)


# bf16 outputs take the segment-state pass, fp16 ones the corrected split (final states formed after the segments)
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("N", [200, 3000])
def test_final_state_may_alias_initial_state(N, out):
    B, H, D = 1, 2, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=7))
    s0 = W.make_state((B,), H, D, D, seed=8).to(DEV)
    ref_o, ref_s = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=out)
    st = s0.clone()
    o, _ = la_prefill(q, k, v, initial_state=st, final_state=st, out_dtype=out)
    torch.cuda.synchronize()
    assert torch.equal(o, ref_o)
    assert torch.equal(st, ref_s)
    _full_compare(q, k, v, s0, torch.bfloat16, o, st)


# slopes decide which chunks the corrected split's correction may skip (their factors below 2^-150)
@pytest.mark.parametrize("out", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("slope_kind", ["zero", "random", "large", "mixed"])
def test_prefill_custom_slopes(slope_kind, out):
    B, N, H, D = 1, 700, 4, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=9))
    rng = np.random.default_rng(0)
    slopes = {"zero": np.zeros(H), "random": rng.uniform(0.0, 1.0, H), "large": np.full(H, 12.0),
              "mixed": np.array([0.0, 0.3, 1.2, 200.0])}[slope_kind]
    sl = torch.tensor(slopes, dtype=torch.float32, device=DEV)
    lam = np.exp(-sl.double().cpu().numpy())
    o, sN = la_prefill(q, k, v, slopes=sl, return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    _full_compare(q, k, v, None, torch.bfloat16, o, sN, lam=lam)


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float16])
def test_state_handoff_chain_equals_one_call(out):
    B, H, D = 1, 2, 128
    lens = [300, 128, 1, 1000]
    N = sum(lens)
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=10))
    st = None
    outs = []
    t = 0
    for L in lens:
        o, st = la_prefill(q[:, t:t + L].contiguous(), k[:, t:t + L].contiguous(), v[:, t:t + L].contiguous(),
                           initial_state=st, return_final_state=True, out_dtype=out)
        outs.append(o)
        t += L
    torch.cuda.synchronize()
    _full_compare(q, k, v, None, torch.bfloat16, torch.cat(outs, 1), st)


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float16])
def test_deterministic(out):
    B, N, H, D = 2, 2500, 4, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=11))
    o1, s1 = la_prefill(q, k, v, return_final_state=True, out_dtype=out)
    o2, s2 = la_prefill(q, k, v, return_final_state=True, out_dtype=out)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


# --------------------------------------------------------------------------- varlen
@pytest.mark.parametrize("dtype, out", [(torch.bfloat16, torch.float16), (torch.bfloat16, torch.float32),
                                        (torch.bfloat16, torch.bfloat16), (torch.float32, torch.float32)])
def test_varlen_ragged_with_guard_bands(dtype, out):
    lens = [0, 1, 127, 128, 129, 700, 3000, 5, 0, 260]
    H, D, pad = 2, 128, 64
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v = (x.to(DEV) for x in W.make_qkv((T,), H, D, dtype=dtype, seed=12))
    s0 = W.make_state((len(lens),), H, D, D, seed=13).to(DEV)
    big = torch.full((T + 2 * pad, H, D), float("nan"), dtype=out, device=DEV)
    o = big[pad:pad + T]
    cu_d = torch.tensor(cu, dtype=torch.int32, device=DEV)
    _, sN = la_prefill_varlen(q, k, v, cu_d, initial_state=s0, return_final_state=True, o=o)
    torch.cuda.synchronize()
    assert torch.isnan(big[:pad].float()).all() and torch.isnan(big[pad + T:].float()).all(), "wrote outside o"
    _full_compare(q, k, v, s0, dtype, o, sN, cu=cu)
    # zero-length sequences pass their state through
    assert torch.equal(sN[0], s0[0]) and torch.equal(sN[8], s0[8])


def test_varlen_equals_separate_calls():
    lens = [513, 64, 1500]
    H, D = 3, 128
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v = (x.to(DEV) for x in W.make_qkv((T,), H, D, seed=14))
    cu_d = torch.tensor(cu, dtype=torch.int32, device=DEV)
    o, sN = la_prefill_varlen(q, k, v, cu_d, return_final_state=True)
    for i, L in enumerate(lens):
        a = int(cu[i])
        oi, si = la_prefill(q[None, a:a + L], k[None, a:a + L], v[None, a:a + L], return_final_state=True)
        torch.cuda.synchronize()
        check(to64(o[a:a + L]), to64(oi[0]), torch.bfloat16, f"seq {i} o", stored_bf16=True)
        check(to64(sN[i]), to64(si[0]), torch.bfloat16, f"seq {i} state")


def test_varlen_malformed_cu_seqlens_is_reported_not_faulted():
    H, D, T = 2, 128, 300
    q, k, v = (x.to(DEV) for x in W.make_qkv((T,), H, D, seed=15))
    cu_d = torch.tensor([0, 200, 100, 300], dtype=torch.int32, device=DEV)   # decreasing
    la_prefill_varlen(q, k, v, cu_d)
    torch.cuda.synchronize()
    assert la_get_device_error() == 1
    from linear_attention_hybrid_b200 import LAError, la_validate_cu_seqlens
    with pytest.raises(LAError):
        la_validate_cu_seqlens(cu_d, T)
    la_validate_cu_seqlens(torch.tensor([0, 100, 300], dtype=torch.int32, device=DEV), T)


# --------------------------------------------------------------------------- decode
@pytest.mark.parametrize("dtype, out, D", [(torch.bfloat16, torch.bfloat16, 128), (torch.bfloat16, torch.float32, 128),
                                           (torch.bfloat16, torch.float16, 128),
                                           (torch.bfloat16, torch.bfloat16, 64), (torch.float32, torch.float32, 128),
                                           (torch.float32, torch.float32, 64)])
def test_decode_steps(dtype, out, D):
    B, H, steps = 3, 5, 6
    S = W.make_state((B,), H, D, D, std=0.1, seed=16).to(DEV)
    S_ref = S.cpu().double().numpy()
    lam = _lam(H)
    for i in range(steps):
        q, k, v = (x.to(DEV) for x in W.make_decode_qkv(B, H, D, step=i, dtype=dtype, seed=16))
        o = la_decode_step(q, k, v, S, out_dtype=out)
        want_o, S_ref = oracle.decode_step(q, k, v, S_ref, lam=lam)
        torch.cuda.synchronize()
        check(to64(o), want_o, dtype, f"step {i} o", stored_bf16=out == torch.bfloat16)
    check(to64(S), S_ref, dtype, "state")


def test_decode_steps_equal_prefill():
    B, N, H, D = 2, 40, 3, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, N), H, D, seed=17))
    s0 = W.make_state((B,), H, D, D, seed=18).to(DEV)
    o_p, s_p = la_prefill(q, k, v, initial_state=s0, return_final_state=True, out_dtype=torch.float32)
    S = s0.clone()
    o_d = torch.stack([la_decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), S,
                                      out_dtype=torch.float32) for t in range(N)], 1)
    torch.cuda.synchronize()
    want_o, want_s = oracle.prefill_recurrent(q, k, v, lam=_lam(H), initial_state=s0.cpu(), return_final_state=True)
    check(to64(o_p), want_o, torch.bfloat16, "prefill o")
    check(to64(o_d), want_o, torch.bfloat16, "decode o")
    check(to64(S), want_s, torch.bfloat16, "decode state")
    check(to64(s_p), want_s, torch.bfloat16, "prefill state")


@pytest.mark.parametrize("dtype, out, D", [(torch.bfloat16, torch.float16, 128), (torch.bfloat16, torch.float32, 64),
                                           (torch.float32, torch.float32, 128)])
@pytest.mark.parametrize("K", [1, 3, 16])
def test_decode_multi_matches_oracle(dtype, out, D, K):
    """K decode steps in one launch equal the oracle's recurrence over those K tokens from the state."""
    B, H = 3, 5
    q, k, v = W.make_qkv((B, K), H, D, dtype=dtype, seed=40 + K)
    S = W.make_state((B,), H, D, D, std=0.1, seed=41).to(DEV)
    want_o, want_s = oracle.prefill_recurrent(q, k, v, lam=_lam(H), initial_state=S.cpu(), return_final_state=True)
    o = la_decode_steps(q.to(DEV), k.to(DEV), v.to(DEV), S, out_dtype=out)
    torch.cuda.synchronize()
    check(to64(o), want_o, dtype, "o")
    check(to64(S), want_s, dtype, "state")


def test_decode_multi_equals_single_steps_exactly():
    """One launch over K tokens performs exactly the arithmetic of K single steps."""
    B, K, H, D = 4, 7, 3, 128
    q, k, v = (x.to(DEV) for x in W.make_qkv((B, K), H, D, seed=42))
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=43).to(DEV)
    S1, S2 = s0.clone(), s0.clone()
    o1 = la_decode_steps(q, k, v, S1, out_dtype=torch.float32)
    o2 = torch.stack([la_decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), S2,
                                     out_dtype=torch.float32) for t in range(K)], 1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    assert torch.equal(S1, S2)


def test_decode_multi_zero_steps_is_a_no_op():
    B, H, D = 2, 3, 128
    S = W.make_state((B,), H, D, D, std=0.1, seed=44).to(DEV)
    before = S.clone()
    x = torch.zeros((B, 0, H, D), dtype=torch.bfloat16, device=DEV)
    la_decode_steps(x, x, x, S)
    torch.cuda.synchronize()
    assert torch.equal(S, before)


# --------------------------------------------------------------------------- the specified workloads at full size
def test_workload_prefill_b4_n4096_sampled():
    wl = W.workloads()["prefill_b4_n4096"]
    q, k, v = W.make_qkv((wl.B, wl.N), wl.H, wl.D, seed=wl.seed, device=DEV)
    o, sN = la_prefill(q, k, v, return_final_state=True, out_dtype=BENCH_OUT)
    torch.cuda.synchronize()
    lam = _lam(wl.H)
    for b, heads in [(0, [0, 15]), (3, [1, 8])]:
        want_o, want_s = oracle_heads(q[b], k[b], v[b], heads, lam)
        check(to64(o[b][:, heads]), want_o, torch.bfloat16, f"b{b} o")
        check(to64(sN[b, heads]), want_s[0], torch.bfloat16, f"b{b} state")


def test_workload_prefill_b4_n4096_d64_sampled():
    """The prefill workload's shape at D = 64, in the launch configuration the benchmark times."""
    wl = W.workloads()["prefill_b4_n4096"]
    D = 64
    q, k, v = W.make_qkv((wl.B, wl.N), wl.H, D, seed=wl.seed + 3, device=DEV)
    o, sN = la_prefill(q, k, v, return_final_state=True, out_dtype=BENCH_OUT)
    torch.cuda.synchronize()
    lam = _lam(wl.H)
    for b, heads in [(0, [0, 15]), (2, [3, 12])]:
        want_o, want_s = oracle_heads(q[b], k[b], v[b], heads, lam)
        check(to64(o[b][:, heads]), want_o, torch.bfloat16, f"b{b} o")
        check(to64(sN[b, heads]), want_s[0], torch.bfloat16, f"b{b} state")


def test_workload_long_n65536_sampled():
    wl = W.workloads()["long_n65536"]
    q, k, v = W.make_qkv((wl.B, wl.N), wl.H, wl.D, seed=wl.seed, device=DEV, k_l2norm=True)
    o, sN = la_prefill(q, k, v, return_final_state=True, out_dtype=BENCH_OUT)
    torch.cuda.synchronize()
    heads = [0, 7, 15]
    want_o, want_s = oracle_heads(q[0], k[0], v[0], heads, _lam(wl.H))
    check(to64(o[0][:, heads]), want_o, torch.bfloat16, "o")
    check(to64(sN[0, heads]), want_s[0], torch.bfloat16, "state")


def test_workload_decode_b256_sampled():
    wl = W.workloads()["decode_b256"]
    steps = wl.steps
    S = W.make_state((wl.B,), wl.H, wl.D, wl.D, std=0.1, seed=wl.seed, device=DEV)
    # 64 (sequence, head) pairs spread over the batch and every head, the first and last of each included
    rng = np.random.default_rng(7)
    picks = [(0, 0), (255, 15), (0, 15), (255, 0)] + [
        (int(b), int(h)) for b, h in zip(rng.choice(np.arange(1, 255), 60, replace=False), np.arange(60) % wl.H)]
    S_ref = np.stack([to64(S[b, h]) for b, h in picks])[None]        # [1, P, D, D]
    lam = _lam(wl.H)[[h for _, h in picks]]
    ib = torch.tensor([b for b, _ in picks], device=DEV)
    ih = torch.tensor([h for _, h in picks], device=DEV)
    for i in range(steps):
        q, k, v = W.make_decode_qkv(wl.B, wl.H, wl.D, step=i, seed=wl.seed, device=DEV)
        o = la_decode_step(q, k, v, S, out_dtype=BENCH_OUT)
        qs, ks, vs = (to64(x[ib, ih])[None] for x in (q, k, v))
        want_o, S_ref = oracle.decode_step(qs, ks, vs, S_ref, lam=lam)
        if i % 10 == 0 or i == steps - 1:
            check(to64(o[ib, ih])[None], want_o, torch.bfloat16, f"step {i} o")
    torch.cuda.synchronize()
    check(to64(S[ib, ih])[None], S_ref, torch.bfloat16, "state after all steps")


def test_workload_varlen_256k_sampled():
    wl = W.workloads()["varlen_256k"]
    lens = list(wl.lengths)
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v = W.make_qkv((T,), wl.H, wl.D, seed=wl.seed, device=DEV)
    cu_d = torch.tensor(cu, dtype=torch.int32, device=DEV)
    o, sN = la_prefill_varlen(q, k, v, cu_d, return_final_state=True, out_dtype=BENCH_OUT)
    torch.cuda.synchronize()
    lam = _lam(wl.H)
    for i, heads in [(0, [0, 15]), (5, [3]), (7, [9])]:
        a, b = int(cu[i]), int(cu[i + 1])
        want_o, want_s = oracle_heads(q[a:b], k[a:b], v[a:b], heads, lam)
        check(to64(o[a:b][:, heads]), want_o, torch.bfloat16, f"seq {i} o")
        check(to64(sN[i, heads]), want_s[0], torch.bfloat16, f"seq {i} state")
    # the 262144-token sequence, run as a chain of 4 calls carrying the state
    N = sum(wl.chain)
    q, k, v = W.make_qkv((1, N), wl.H, wl.D, seed=wl.seed + 1, device=DEV)
    st, outs, t = None, [], 0
    for L in wl.chain:
        oc, st = la_prefill(q[:, t:t + L].contiguous(), k[:, t:t + L].contiguous(), v[:, t:t + L].contiguous(),
                            initial_state=st, return_final_state=True, out_dtype=BENCH_OUT)
        outs.append(oc)
        t += L
    torch.cuda.synchronize()
    heads = [0, 15]
    want_o, want_s = oracle_heads(q[0], k[0], v[0], heads, lam)
    check(to64(torch.cat(outs, 1)[0][:, heads]), want_o, torch.bfloat16, "chain o")
    check(to64(st[0, heads]), want_s[0], torch.bfloat16, "chain state")
