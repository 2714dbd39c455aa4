"""Randomised GPU parity: seeded draws of shape, dtype, output type, states, decay slopes and varlen layout,
each run through the library and compared with the oracle under the operator's bound. They reach plan
corners the hand-picked cases may miss (segment counts, chunks cut by segment and sequence ends, empty
sequences next to long ones, heads that do not divide the SM count)."""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_hybrid_b200 import (la_get_device_error, la_prefill, la_prefill_backward, la_prefill_varlen,
                                          la_prefill_varlen_backward)
from linear_attention_hybrid_b200 import inputs as W
from tests.parity_util import check, to64

pytestmark = pytest.mark.gpu
DEV = "cuda"
CASES = 40


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def _draw(seed):
    rng = np.random.default_rng(1000 + seed)
    D = 64 if rng.random() < 0.15 else 128
    fp32 = rng.random() < 0.15
    dtype = torch.float32 if fp32 else torch.bfloat16
    out = torch.float32 if fp32 else [torch.float16, torch.float32, torch.bfloat16][rng.integers(3)]
    H = int(rng.integers(1, 21))
    varlen = rng.random() < 0.4
    budget = 60000 // H  # tokens, so that the oracle stays fast
    if varlen:
        nseq = int(rng.integers(1, 7))
        lens = [int(x) for x in rng.integers(0, max(2, budget // nseq), nseq)]
        if rng.random() < 0.3:
            lens[int(rng.integers(nseq))] = 0
        B, N = nseq, None
    else:
        B = int(rng.integers(1, 5))
        N = int(rng.integers(1, max(2, budget // B)))
        lens = None
    states = rng.random() < 0.6
    slopes = rng.uniform(0.0, 3.0, H) if rng.random() < 0.3 else None
    return dict(D=D, dtype=dtype, out=out, H=H, B=B, N=N, lens=lens, states=states, slopes=slopes)


def _lam(c):
    return oracle.decay(c["H"]) if c["slopes"] is None else np.exp(-np.asarray(c["slopes"], np.float64))


def _slopes_dev(c):
    return None if c["slopes"] is None else torch.tensor(c["slopes"], dtype=torch.float32, device=DEV)


@pytest.mark.parametrize("seed", range(CASES))
def test_random_prefill(seed):
    c = _draw(seed)
    H, D = c["H"], c["D"]
    if c["lens"] is None:
        q, k, v = W.make_qkv((c["B"], c["N"]), H, D, dtype=c["dtype"], seed=seed)
        nseq, cu = c["B"], None
    else:
        cu = W.cu_seqlens_of(c["lens"])
        q, k, v = W.make_qkv((int(cu[-1]),), H, D, dtype=c["dtype"], seed=seed)
        nseq = len(c["lens"])
    s0 = W.make_state((nseq,), H, D, D, std=0.1, seed=seed + 1) if c["states"] else None
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    s0d = None if s0 is None else s0.to(DEV)
    if cu is None:
        o, sN = la_prefill(qd, kd, vd, initial_state=s0d, return_final_state=True, slopes=_slopes_dev(c),
                           out_dtype=c["out"])
    else:
        o, sN = la_prefill_varlen(qd, kd, vd, torch.tensor(cu, dtype=torch.int32, device=DEV), initial_state=s0d,
                                  return_final_state=True, slopes=_slopes_dev(c), out_dtype=c["out"])
    torch.cuda.synchronize()
    want_o, want_s = oracle.prefill_recurrent(q, k, v, cu_seqlens=cu, lam=_lam(c), initial_state=s0,
                                              return_final_state=True)
    check(to64(o), want_o, c["dtype"], f"o {c}", stored_bf16=c["out"] == torch.bfloat16)
    check(to64(sN).reshape(want_s.shape), want_s, c["dtype"], f"final state {c}")


@pytest.mark.parametrize("seed", range(CASES // 2))
def test_random_backward(seed):
    c = _draw(100 + seed)
    H, D = c["H"], c["D"]
    if c["lens"] is None:
        lead, nseq, cu = (c["B"], c["N"]), c["B"], None
    else:
        cu = W.cu_seqlens_of(c["lens"])
        lead, nseq = (int(cu[-1]),), len(c["lens"])
    q, k, v = W.make_qkv(lead, H, D, dtype=c["dtype"], seed=seed)
    g = W.make_grad_out(lead, H, D, dtype=c["dtype"], seed=seed + 7)
    s0 = W.make_state((nseq,), H, D, D, std=0.1, seed=seed + 1) if c["states"] else None
    dsn = W.make_state((nseq,), H, D, D, std=0.1, seed=seed + 2) if c["states"] else None
    dev = [x.to(DEV) for x in (q, k, v, g)]
    kw = dict(initial_state=None if s0 is None else s0.to(DEV), d_final_state=None if dsn is None else dsn.to(DEV),
              return_d_initial_state=True, slopes=_slopes_dev(c), out_dtype=c["out"])
    if cu is None:
        got = la_prefill_backward(*dev, **kw)
    else:
        got = la_prefill_varlen_backward(*dev, torch.tensor(cu, dtype=torch.int32, device=DEV), **kw)
    torch.cuda.synchronize()
    want = oracle.prefill_backward_recurrent(q, k, v, g, cu_seqlens=cu, lam=_lam(c), initial_state=s0,
                                             d_final_state=dsn)
    for name, a, b in zip(("dq", "dk", "dv"), got[:3], want[:3]):
        check(to64(a), b, c["dtype"], f"{name} {c}", stored_bf16=c["out"] == torch.bfloat16)
    check(to64(got[3]).reshape(want[3].shape), want[3], c["dtype"], f"d_initial_state {c}")
