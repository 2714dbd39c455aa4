"""GPU parity of the backward pass (la_prefill_backward, la_prefill_varlen_backward) against the
oracle's gradients (the adjoint of the recurrence, fp64).

Every gradient is held to the operator's bound against its own RMS: bf16 inputs max|err| <= 2e-2 *
RMS (plus half a bf16 ulp of the value when the gradient is stored as bf16), fp32 inputs
max|err| <= 1e-4 * min(1, RMS). dS_0 is an fp32 state and is held to the same rule.
"""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_hybrid_b200 import (la_get_device_error, la_last_launch_count, la_prefill_backward,
                                          la_prefill_varlen_backward)
from linear_attention_hybrid_b200 import inputs as W
from tests.parity_util import check, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def _inputs(lead, H, D, dtype=torch.bfloat16, seed=0, states=True, nstate=None):
    q, k, v = W.make_qkv(lead, H, D, dtype=dtype, seed=seed)
    g = W.make_grad_out(lead, H, D, dtype=dtype, seed=seed + 1000)
    ns = (lead[0],) if nstate is None else (nstate,)
    s0 = W.make_state(ns, H, D, D, std=0.1, seed=seed + 2000) if states else None
    dsn = W.make_state(ns, H, D, D, std=0.1, seed=seed + 3000) if states else None
    return q, k, v, g, s0, dsn


def _dev(*xs):
    return [None if x is None else x.to(DEV) for x in xs]


def _compare(got, q, k, v, g, s0, dsn, dtype, lam=None, cu=None):
    """got = (dq, dk, dv, ds0) from the GPU; the oracle runs on the same (CPU) inputs."""
    H = q.shape[-2]
    lam = oracle.decay(H) if lam is None else lam
    want = oracle.prefill_backward_recurrent(q, k, v, g, cu_seqlens=cu, lam=lam, initial_state=s0,
                                             d_final_state=dsn)
    for name, a, b in zip(("dq", "dk", "dv"), got[:3], want[:3]):
        check(to64(a), b, dtype, name, stored_bf16=a.dtype == torch.bfloat16)
    if len(got) > 3 and got[3] is not None:
        check(to64(got[3]).reshape(want[3].shape), want[3], dtype, "d_initial_state")


# --------------------------------------------------------------------------- tensor-core path
@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 300, 1000, 2177])
@pytest.mark.parametrize("with_states", [False, True])
@pytest.mark.parametrize("out", [torch.float16, torch.float32, torch.bfloat16])
def test_backward_bf16_ragged(N, with_states, out):
    B, H, D = 2, 3, 128
    q, k, v, g, s0, dsn = _inputs((B, N), H, D, seed=N, states=with_states)
    got = la_prefill_backward(*_dev(q, k, v, g), initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                              return_d_initial_state=True, out_dtype=out)
    torch.cuda.synchronize()
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16)


@pytest.mark.parametrize("B, N, H", [(1, 8192, 2), (1, 6000, 4), (2, 3333, 8)])
def test_backward_segmented(B, N, H):
    """Long sequences over few heads: many segments, the state pass over fine units in both directions."""
    q, k, v, g, s0, dsn = _inputs((B, N), H, 128, seed=N + H)
    got = la_prefill_backward(*_dev(q, k, v, g), initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                              return_d_initial_state=True)
    torch.cuda.synchronize()
    assert la_last_launch_count() == 2 + 3 * 2   # two transposes; state pass + chunk kernel per sweep
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16)


def test_backward_prefill_workload_sampled():
    """The prefill workload's shape (B=4, N=4096, H=16: two segments per sequence, the long one first in the
    forward sweep and last in the backward sweeps); sampled (sequence, head) slices, each whole."""
    B, N, H, D = 4, 4096, 16, 128
    q, k, v, g, s0, dsn = _inputs((B, N), H, D, seed=0)
    got = la_prefill_backward(*_dev(q, k, v, g), initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                              return_d_initial_state=True, out_dtype=torch.float16)
    torch.cuda.synchronize()
    lam = oracle.decay(H)
    for b in (0, 3):
        hs = [0, 7, 15]
        sl = lambda x: x[b:b + 1][:, :, hs]  # noqa: E731
        want = oracle.prefill_backward_recurrent(sl(q), sl(k), sl(v), sl(g), lam=lam[hs],
                                                 initial_state=s0[b:b + 1, hs], d_final_state=dsn[b:b + 1, hs])
        for name, a, w in zip(("dq", "dk", "dv"), got[:3], want[:3]):
            check(to64(a[b:b + 1][:, :, hs]), w, torch.bfloat16, f"{name} seq {b}")
        check(to64(got[3][b:b + 1, hs]), want[3], torch.bfloat16, f"d_initial_state seq {b}")


@pytest.mark.parametrize("B, N, H", [(4, 1000, 14), (3, 1337, 20)])
def test_backward_dv_first(B, N, H):
    """50..74 (sequence, head) pairs in a uniform batch: the dv sweep runs first with the whole GPU's segmented
    plan, then the dq and dk sweeps unsegmented; d_initial_state is written over d_final_state in place."""
    q, k, v, g, s0, dsn = _inputs((B, N), H, 128, seed=B * N + H)
    qd, kd, vd, gd = _dev(q, k, v, g)
    ds = _dev(dsn)[0].clone()
    got = la_prefill_backward(qd, kd, vd, gd, initial_state=_dev(s0)[0], d_final_state=ds, d_initial_state=ds)
    torch.cuda.synchronize()
    assert got[3].data_ptr() == ds.data_ptr()
    assert la_last_launch_count() == 2 + 2 + 1 + 1   # transposes; dv: state pass + chunk kernel; dq, dk: chunk kernel
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16)


@pytest.mark.parametrize("B, N, H", [(1, 6000, 4), (4, 1000, 14)])
def test_backward_d64_tensor_core(B, N, H):
    """D = 64 with bf16 inputs: the three sweeps run the chunk kernel's D = 64 instance (and the zero-padded
    segment-state kernel)."""
    q, k, v, g, s0, dsn = _inputs((B, N), H, 64, seed=B * N + H + 1)
    got = la_prefill_backward(*_dev(q, k, v, g), initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                              return_d_initial_state=True)
    torch.cuda.synchronize()
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16)


def test_backward_unsegmented_launches():
    B, N, H, D = 10, 300, 16, 128   # B*H >= 148: one unit per (sequence, head)
    q, k, v, g, _, _ = _inputs((B, N), H, D, seed=3, states=False)
    got = la_prefill_backward(*_dev(q, k, v, g))
    torch.cuda.synchronize()
    assert la_last_launch_count() == 3   # one chunk kernel per sweep, no transposes without states
    _compare(got, q, k, v, g, None, None, torch.bfloat16)


# --------------------------------------------------------------------------- fp32 (CUDA cores) and bf16 D = 64 (its own instances)
@pytest.mark.parametrize("dtype, out, D", [(torch.float32, torch.float32, 128), (torch.float32, torch.float32, 64),
                                           (torch.bfloat16, torch.bfloat16, 64), (torch.bfloat16, torch.float32, 64)])
@pytest.mark.parametrize("N", [1, 63, 64, 65, 300])
def test_backward_fp32_and_d64_paths(dtype, out, D, N):
    B, H = 2, 3
    q, k, v, g, s0, dsn = _inputs((B, N), H, D, dtype=dtype, seed=N + D)
    got = la_prefill_backward(*_dev(q, k, v, g), initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                              return_d_initial_state=True, out_dtype=out)
    torch.cuda.synchronize()
    _compare(got, q, k, v, g, s0, dsn, dtype)


# --------------------------------------------------------------------------- edge cases
def test_backward_zero_length_passes_state_gradient_through():
    B, N, H, D = 2, 0, 3, 128
    q = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=DEV)
    dsn = W.make_state((B,), H, D, D, seed=6).to(DEV)
    dq, dk, dv, ds0 = la_prefill_backward(q, q.clone(), q.clone(), q.clone(), d_final_state=dsn,
                                          return_d_initial_state=True)
    torch.cuda.synchronize()
    assert dq.numel() == 0 and torch.equal(ds0, dsn)


def test_backward_without_state_gradient_has_zero_state_term():
    B, N, H, D = 1, 700, 2, 128
    q, k, v, g, _, _ = _inputs((B, N), H, D, seed=21, states=False)
    got = la_prefill_backward(*_dev(q, k, v, g), return_d_initial_state=True)
    torch.cuda.synchronize()
    _compare(got, q, k, v, g, None, None, torch.bfloat16)


@pytest.mark.parametrize("N", [200, 3000])
@pytest.mark.parametrize("alias", ["d_final_state", "initial_state"])
def test_d_initial_state_may_alias(N, alias):
    B, H, D = 1, 2, 128
    q, k, v, g, s0, dsn = _inputs((B, N), H, D, seed=N + 7)
    qd, kd, vd, gd, s0d, dsnd = _dev(q, k, v, g, s0, dsn)
    ref = la_prefill_backward(qd, kd, vd, gd, initial_state=s0d, d_final_state=dsnd, return_d_initial_state=True)
    buf = (dsnd if alias == "d_final_state" else s0d).clone()
    kw = dict(initial_state=s0d, d_final_state=dsnd)
    kw[alias] = buf
    got = la_prefill_backward(qd, kd, vd, gd, d_initial_state=buf, **kw)
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16)


@pytest.mark.parametrize("slope_kind", ["zero", "random", "large"])
def test_backward_custom_slopes(slope_kind):
    B, N, H, D = 1, 700, 4, 128
    q, k, v, g, s0, dsn = _inputs((B, N), H, D, seed=9)
    rng = np.random.default_rng(0)
    slopes = {"zero": np.zeros(H), "random": rng.uniform(0.0, 1.0, H), "large": np.full(H, 12.0)}[slope_kind]
    sl = torch.tensor(slopes, dtype=torch.float32, device=DEV)
    lam = np.exp(-sl.double().cpu().numpy())
    got = la_prefill_backward(*_dev(q, k, v, g), initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                              return_d_initial_state=True, slopes=sl)
    torch.cuda.synchronize()
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16, lam=lam)


def test_backward_deterministic():
    B, N, H, D = 2, 2500, 4, 128
    q, k, v, g, s0, dsn = _dev(*_inputs((B, N), H, D, seed=11))
    a = la_prefill_backward(q, k, v, g, initial_state=s0, d_final_state=dsn, return_d_initial_state=True)
    b = la_prefill_backward(q, k, v, g, initial_state=s0, d_final_state=dsn, return_d_initial_state=True)
    torch.cuda.synchronize()
    for x, y in zip(a, b):
        assert torch.equal(x, y)


# --------------------------------------------------------------------------- varlen
@pytest.mark.parametrize("dtype, out", [(torch.bfloat16, torch.float16), (torch.bfloat16, torch.bfloat16),
                                        (torch.float32, torch.float32)])
def test_backward_varlen_ragged_with_guard_bands(dtype, out):
    lens = [0, 1, 127, 128, 129, 700, 3000, 5, 0, 260]
    H, D, pad = 2, 128, 64
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v, g, s0, dsn = _inputs((T,), H, D, dtype=dtype, seed=12, nstate=len(lens))
    bigs = [torch.full((T + 2 * pad, H, D), float("nan"), dtype=out, device=DEV) for _ in range(3)]
    dq, dk, dv = (b[pad:pad + T] for b in bigs)
    cu_d = torch.tensor(cu, dtype=torch.int32, device=DEV)
    got = la_prefill_varlen_backward(*_dev(q, k, v, g), cu_d, initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                                     return_d_initial_state=True, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    for b in bigs:
        assert torch.isnan(b[:pad].float()).all() and torch.isnan(b[pad + T:].float()).all(), "wrote outside"
    _compare(got, q, k, v, g, s0, dsn, dtype, cu=cu)
    # zero-length sequences pass the state gradient through
    assert torch.equal(got[3][0].cpu(), dsn[0]) and torch.equal(got[3][8].cpu(), dsn[8])


def test_backward_varlen_long_sequences_segmented():
    lens = [9000, 300, 5000]
    H, D = 2, 128
    cu = W.cu_seqlens_of(lens)
    T = int(cu[-1])
    q, k, v, g, s0, dsn = _inputs((T,), H, D, seed=15, nstate=len(lens))
    cu_d = torch.tensor(cu, dtype=torch.int32, device=DEV)
    got = la_prefill_varlen_backward(*_dev(q, k, v, g), cu_d, initial_state=_dev(s0)[0], d_final_state=_dev(dsn)[0],
                                     return_d_initial_state=True, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _compare(got, q, k, v, g, s0, dsn, torch.bfloat16, cu=cu)
