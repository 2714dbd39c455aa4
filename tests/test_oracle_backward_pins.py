"""Pins for the oracle's backward pass: checks against things other than the backward codings.

The pages do not treat the backward pass; the oracle's gradients are the derivative
of the operator's definition. They are pinned to the FORWARD oracle (already pinned
by tests/test_oracle_pins.py) through an identity that holds exactly: the loss
L = <dO, o> + <dS_N, S_N> is linear in each of q, k, v and S0 on its own, so for any
perturbation d of one of them L(x + d) - L(x) = <dL/dx, d> up to fp64 rounding (no
finite-difference error). Beside that: the three codings agree, a single token and
lambda = 1 have closed forms, the reverse-time reading (dv is a forward pass over the
reversed sequence) holds, and planted mistakes are caught.
"""

import numpy as np
import pytest

import oracle

BWD_FORMS = [oracle.prefill_backward_recurrent, oracle.prefill_backward_quadratic,
             oracle.prefill_backward_bruteforce]


def _close(a, b, rtol):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rtol * scale, f"max|err| {err:.3e} > {rtol:.1e} * {scale:.3e}"


def _inputs(seed, T, H, D, nseq=1):
    rng = np.random.default_rng(seed)
    q, k, v, g = (rng.standard_normal((T, H, D)) for _ in range(4))
    s0 = rng.standard_normal((nseq, H, D, D))
    dsn = rng.standard_normal((nseq, H, D, D))
    lam = rng.uniform(0.2, 1.0, H)
    return q, k, v, g, s0, dsn, lam


def _loss(q, k, v, g, s0, dsn, lam, cu=None):
    o, sN = oracle.prefill_recurrent(q, k, v, cu_seqlens=cu, lam=lam, initial_state=s0, return_final_state=True)
    return float(np.sum(g * o) + np.sum(dsn * sN))


# --------------------------------------------------------------------------- codings agree
@pytest.mark.parametrize("T", [1, 2, 17, 40])
@pytest.mark.parametrize("with_states", [False, True])
def test_three_backward_forms_agree(T, with_states):
    q, k, v, g, s0, dsn, lam = _inputs(T, T, 2, 3)
    kw = dict(lam=lam, initial_state=s0 if with_states else None, d_final_state=dsn if with_states else None)
    want = oracle.prefill_backward_bruteforce(q, k, v, g, **kw)
    for form in BWD_FORMS[:2]:
        for a, b in zip(form(q, k, v, g, **kw), want):
            _close(a, b, 1e-12)


def test_backward_forms_agree_varlen_with_empty_sequence():
    cu = [0, 5, 5, 19, 30]
    q, k, v, g, s0, dsn, lam = _inputs(3, 30, 2, 4, nseq=4)
    kw = dict(cu_seqlens=cu, lam=lam, initial_state=s0, d_final_state=dsn)
    want = oracle.prefill_backward_bruteforce(q, k, v, g, **kw)
    for form in BWD_FORMS[:2]:
        for a, b in zip(form(q, k, v, g, **kw), want):
            _close(a, b, 1e-12)
    # an empty sequence passes the state gradient through: dS_0 = dS_N
    _close(want[3][1], dsn[1], 0)


# --------------------------------------------------------------------------- exact adjoint identity
@pytest.mark.parametrize("which", ["q", "k", "v", "s0"])
@pytest.mark.parametrize("cu", [None, [0, 13, 13, 50]])
def test_gradient_is_the_exact_directional_derivative_of_the_forward(which, cu):
    """L is linear in each input on its own, so L(x + d) - L(x) equals <grad, d> exactly."""
    nseq = 1 if cu is None else len(cu) - 1
    q, k, v, g, s0, dsn, lam = _inputs(7, 50, 3, 5, nseq=nseq)
    dq, dk, dv, ds0 = oracle.prefill_backward_recurrent(q, k, v, g, cu_seqlens=cu, lam=lam, initial_state=s0,
                                                        d_final_state=dsn)
    args = dict(q=q, k=k, v=v, s0=s0)
    grad = dict(q=dq, k=dk, v=dv, s0=ds0)[which]
    d = np.random.default_rng(8).standard_normal(args[which].shape)
    base = _loss(q, k, v, g, s0, dsn, lam, cu)
    args[which] = args[which] + d
    moved = _loss(args["q"], args["k"], args["v"], g, args["s0"], dsn, lam, cu)
    want = float(np.sum(grad * d))
    assert abs((moved - base) - want) <= 1e-10 * max(1.0, abs(want), abs(base))


def test_gradient_of_final_state_alone():
    """With dO = 0 only the final state carries gradient: dq = 0, and dk, dv, dS_0 follow from
    S_N = lambda^n S0 + sum_s lambda^(n-1-s) k_s^T v_s by hand."""
    q, k, v, _, s0, dsn, lam = _inputs(9, 12, 2, 3)
    g = np.zeros_like(q)
    dq, dk, dv, ds0 = oracle.prefill_backward_recurrent(q, k, v, g, lam=lam, initial_state=s0, d_final_state=dsn)
    assert np.count_nonzero(dq) == 0
    n = q.shape[0]
    for h in range(2):
        u = lam[h] ** (n - 1 - np.arange(n))
        _close(dk[:, h], u[:, None] * (v[:, h] @ dsn[0, h].T), 1e-13)
        _close(dv[:, h], u[:, None] * (k[:, h] @ dsn[0, h]), 1e-13)
        _close(ds0[0, h], lam[h] ** n * dsn[0, h], 1e-14)


# --------------------------------------------------------------------------- closed forms
def test_single_token_closed_form():
    """N = 1: o = q (lambda S0 + k^T v), S_1 = lambda S0 + k^T v, so with G = q^T dO + dS_N:
    dq = (lambda S0 + k^T v) dO, dk = G v, dv = k G, dS_0 = lambda G."""
    q, k, v, g, s0, dsn, lam = _inputs(4, 1, 1, 4)
    dq, dk, dv, ds0 = oracle.prefill_backward_recurrent(q, k, v, g, lam=lam, initial_state=s0, d_final_state=dsn)
    S1 = lam[0] * s0[0, 0] + np.outer(k[0, 0], v[0, 0])
    G = np.outer(q[0, 0], g[0, 0]) + dsn[0, 0]
    _close(dq[0, 0], S1 @ g[0, 0], 1e-14)
    _close(dk[0, 0], G @ v[0, 0], 1e-14)
    _close(dv[0, 0], k[0, 0] @ G, 1e-14)
    _close(ds0[0, 0], lam[0] * G, 1e-14)


def test_lambda_one_is_causal_linear_attention_gradient():
    """lambda = 1: O = tril(Q K^T) V, whose gradients are dQ = tril(dO V^T) K, dK = tril(dO V^T)^T Q,
    dV = tril(Q K^T)^T dO (textbook causal linear attention)."""
    q, k, v, g, _, _, _ = _inputs(5, 23, 1, 4)
    dq, dk, dv, _ = oracle.prefill_backward_recurrent(q, k, v, g, lam=[1.0])
    Q, K, V, G = q[:, 0], k[:, 0], v[:, 0], g[:, 0]
    E = np.tril(G @ V.T)
    _close(dq[:, 0], E @ K, 1e-12)
    _close(dk[:, 0], E.T @ Q, 1e-12)
    _close(dv[:, 0], np.tril(Q @ K.T).T @ G, 1e-12)


def test_dv_is_a_forward_pass_over_the_reversed_sequence():
    """Reverse-time reading: with the sequence reversed, dv is the forward operator with q <- k,
    k <- q, v <- dO and initial state dS_N / lambda (the state gradient enters before the last token)."""
    q, k, v, g, _, dsn, lam = _inputs(6, 31, 2, 4)
    _, _, dv, _ = oracle.prefill_backward_recurrent(q, k, v, g, lam=lam, d_final_state=dsn)
    rev = slice(None, None, -1)
    fwd = oracle.prefill_recurrent(k[rev], q[rev], g[rev], lam=lam, initial_state=dsn / lam[None, :, None, None])
    _close(dv, fwd[rev], 1e-12)


# --------------------------------------------------------------------------- planted mistakes
def _mutant(kind):
    """The matrix-form gradients of one sequence with one plausible mistake planted in them."""
    def f(q, k, v, g, lam, s0, dsn):
        n, H, _ = q.shape
        t = np.arange(n)
        d = (t[:, None] - t[None, :]).astype(float)
        out = [np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(s0)]
        for h in range(H):
            lh = lam[h]
            M = np.where(d >= 0, lh ** np.maximum(d, 0), 0.0)
            if kind == "mask_not_transposed_for_dk":
                Mk = M
            else:
                Mk = M.T
            Q, K, V, G = q[:, h], k[:, h], v[:, h], g[:, h]
            w = lh ** (t + 1.0)
            u = lh ** (n - 1.0 - t)
            if kind == "state_decay_off_by_one":
                u = lh ** (n - t + 0.0)
            E = (G @ V.T) * M
            out[0][:, h] = E @ K + w[:, None] * (G @ (s0[0, h] if kind == "s0_not_transposed" else s0[0, h].T))
            out[1][:, h] = (((G @ V.T).T * Mk) @ Q) + u[:, None] * (V @ dsn[0, h].T)
            out[2][:, h] = ((Q @ K.T) * M).T @ G + u[:, None] * (K @ dsn[0, h])
            ds0 = Q.T @ (w[:, None] * G) + lh ** n * dsn[0, h]
            if kind == "ds0_missing_decay":
                ds0 = Q.T @ G + lh ** n * dsn[0, h]
            out[3][0, h] = ds0
        return out
    return f


@pytest.mark.parametrize("kind", ["mask_not_transposed_for_dk", "state_decay_off_by_one", "s0_not_transposed",
                                  "ds0_missing_decay"])
def test_backward_pins_catch_planted_mistakes(kind):
    q, k, v, g, s0, dsn, lam = _inputs(12, 20, 2, 3)
    grads = _mutant(kind)(q, k, v, g, lam, s0, dsn)
    base = _loss(q, k, v, g, s0, dsn, lam)
    caught = False
    for idx, name in enumerate(["q", "k", "v", "s0"]):
        args = dict(q=q, k=k, v=v, s0=s0)
        d = np.random.default_rng(idx).standard_normal(args[name].shape)
        args[name] = args[name] + d
        moved = _loss(args["q"], args["k"], args["v"], g, args["s0"], dsn, lam)
        if abs((moved - base) - float(np.sum(grads[idx] * d))) > 1e-9 * max(1.0, abs(base)):
            caught = True
    assert caught, f"planted mistake {kind!r} was not caught"
    # the unmutated coding passes the same identity
    good = _mutant("none")(q, k, v, g, lam, s0, dsn)
    for a, b in zip(good, oracle.prefill_backward_recurrent(q, k, v, g, lam=lam, initial_state=s0,
                                                            d_final_state=dsn)):
        _close(a, b, 1e-12)


# --------------------------------------------------------------------------- context-parallel backward
def test_sharded_backward_equals_one_backward():
    """The context-parallel reading of the backward pass: shard r runs its local backward from the forward
    state entering it, S_in,r = sum_{r'<r} lambda^((r-1-r')L) dS_r' + lambda^(rL) S0 (dS_r' the shard states
    from a zero start), and from the reversed state entering it from the right,
    H_in,r = sum_{r'>r} lambda^((r'-r-1)L) dH_r' + lambda^((R-1-r)L) dS_N, with dH_r' = sum_s lambda^(s+1)
    q_s^T dO_s over shard r' (its local backward's dS_0 from a zero state gradient). The shards' dq, dk,
    dv are the whole backward's, and shard 0's dS_0 is the whole dS_0."""
    L, R, H, D = 23, 4, 2, 5
    q, k, v, g, s0, dsn, lam = _inputs(21, L * R, H, D)
    want = oracle.prefill_backward_recurrent(q, k, v, g, lam=lam, initial_state=s0, d_final_state=dsn)
    sl = [slice(r * L, (r + 1) * L) for r in range(R)]
    dS = [oracle.prefill_recurrent(q[x], k[x], v[x], lam=lam, return_final_state=True)[1][0] for x in sl]
    dH = [oracle.prefill_backward_recurrent(q[x], k[x], v[x], g[x], lam=lam)[3][0] for x in sl]
    lamL = (lam ** L)[:, None, None]
    got = []
    for r in range(R):
        S_in = lamL ** r * s0[0] + sum(lamL ** (r - 1 - rp) * dS[rp] for rp in range(r))
        H_in = lamL ** (R - 1 - r) * dsn[0] + sum(lamL ** (rp - r - 1) * dH[rp] for rp in range(r + 1, R))
        got.append(oracle.prefill_backward_recurrent(q[sl[r]], k[sl[r]], v[sl[r]], g[sl[r]], lam=lam,
                                                     initial_state=S_in[None], d_final_state=H_in[None]))
    for i in range(3):
        _close(np.concatenate([x[i] for x in got]), want[i], 1e-11)
    _close(got[0][3], want[3], 1e-11)
