"""Helpers shared by the GPU parity tests: the tolerance rule and oracle runs
on sampled (sequence, head) slices.

Tolerance (the operator spec): bf16 inputs pass when max|err| <= 2e-2 * RMS of
the oracle's values over the compared elements; fp32 inputs when
max|err| <= 1e-4 * min(1, RMS). Final states (always fp32) use the same rule
against the RMS of the oracle's state.

The bound is on the computed result. When the result is stored as bf16, its
own rounding is not computation error, yet alone it reaches ~0.016-0.023 RMS
on large Gaussian-like outputs. A stored value g = rn_bf16(c) only tells that
the kernel's fp32 result c lies within half a bf16 ulp of g, so the test asks
for what that permits and no more: |g - want| <= bound + ulp_bf16(g) / 2, i.e.
that some c rounding to g is within the bound. (Comparing g with
rn_bf16(want) instead would fail correct results whenever c and want fall on
either side of a rounding boundary: one bf16 ulp of a 5-sigma value is ~0.04
RMS.) The benchmarked configuration stores o as fp16 and is held to the bare
bound with no allowance.
"""

import numpy as np
import torch

import oracle

BF16_REL = 2e-2
FP32_REL = 1e-4


def to64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_half_ulp(x):
    """Half the spacing of bf16 values at each element of x (8 significant bits; bf16 shares fp32's exponent
    range, so for |x| below 2^-126 the spacing is that of the subnormals, 2^-133)."""
    ax = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(ax > 0, np.exp2(e - 8.0), 2.0 ** -134)


def check(got, want, dtype, what="", stored_bf16=False):
    """dtype: input dtype (selects the bound); stored_bf16: `got` was stored as bf16."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    if want.size == 0:
        return 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    rms = float(np.sqrt(np.mean(want ** 2)))
    diff = np.abs(got - want)
    if stored_bf16:
        diff = np.maximum(diff - bf16_half_ulp(got), 0.0)
    err = float(np.max(diff))
    if dtype == torch.float32:
        bound = FP32_REL * min(1.0, rms)
    else:
        bound = BF16_REL * rms
    assert err <= bound, f"{what}: max|err| {err:.3e} > bound {bound:.3e} (rms {rms:.3e})"
    return err / max(rms, 1e-300)


def oracle_heads(q, k, v, heads, lam, s0=None, want_state=True):
    """Oracle (recurrent form, all host cores) for one sequence [N, H, D] on a subset of heads."""
    hs = list(heads)
    qs, ks, vs = (to64(x[:, hs, :]) for x in (q, k, v))
    s0s = None if s0 is None else to64(s0[hs]).reshape(1, len(hs), *s0.shape[-2:])
    return oracle.prefill_recurrent(qs, ks, vs, lam=np.asarray(lam)[hs], initial_state=s0s,
                                    return_final_state=want_state)
