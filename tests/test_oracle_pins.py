"""Pins for the oracle: checks against things other than the oracle itself.

The report pages (Ling & Ring 2.6 Technical Report) print no operator values,
so the oracle is pinned by mathematics: hand-worked examples
(tests/golden/worked_examples.json), closed forms (lambda = 1 cumulative sum,
constant inputs as a geometric series, impulse response), special cases, the
three independent codings agreeing, and the composition invariants the pages
rely on (section "Long-Context Training: Context Parallel for Lightning
Attention": a sequence can be split into shards computed from a zero state and
corrected with the states of earlier shards; varlen packing keeps sequences
independent). A planted-mistake test at the end shows that the pins catch the
plausible errors.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")
RTOL = 1e-12


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _close(a, b, rtol=RTOL):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    assert a.shape == b.shape, (a.shape, b.shape)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rtol * scale, f"max|err| {err:.3e} > {rtol:.1e} * {scale:.3e}"


ALL_FORMS = [oracle.prefill_recurrent, oracle.prefill_quadratic, oracle.prefill_bruteforce]


# --------------------------------------------------------------------------- hand-worked examples
def _golden_cases():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("form", ALL_FORMS, ids=lambda f: f.__name__)
@pytest.mark.parametrize("case", _golden_cases()["cases"], ids=lambda c: c["name"])
def test_worked_examples(form, case):
    q, k, v = (np.array(case[x], np.float64) for x in ("q", "k", "v"))
    s0 = None if case["initial_state"] is None else np.array(case["initial_state"], np.float64)
    o, sN = form(q, k, v, cu_seqlens=case.get("cu_seqlens"), lam=case["lam"], initial_state=s0,
                 return_final_state=True)
    _close(o, np.array(case["o"], np.float64), 1e-15)
    _close(sN, np.array(case["final_state"], np.float64), 1e-15)


def test_worked_examples_by_decode_steps():
    for case in _golden_cases()["cases"]:
        if case.get("cu_seqlens") is not None:
            continue
        q, k, v = (np.array(case[x], np.float64) for x in ("q", "k", "v"))
        T, H, Dk = q.shape
        S = np.zeros((1, H, Dk, v.shape[2])) if case["initial_state"] is None else np.array(case["initial_state"])
        for t in range(T):
            o, S = oracle.decode_step(q[t:t + 1], k[t:t + 1], v[t:t + 1], S, lam=case["lam"])
            _close(o[0], np.array(case["o"][t]), 1e-15)
        _close(S, np.array(case["final_state"]), 1e-15)


_CLOSED = {"exp(-1/sqrt(2))": math.exp(-1.0 / math.sqrt(2.0)), "exp(-1/16)": math.exp(-1.0 / 16.0),
           "exp(-1/256)": math.exp(-1.0 / 256.0)}


def test_decay_schedule_closed_forms():
    for row in _golden_cases()["decay_schedule"]["values"]:
        lam = oracle.decay(row["H"])
        assert lam.shape == (row["H"],)
        assert abs(lam[row["h"]] - _CLOSED[row["closed_form"]]) <= 1e-15


def test_decay_schedule_monotone_in_unit_interval():
    for H in (1, 2, 3, 16, 64):
        lam = oracle.decay(H)
        assert np.all(lam > 0) and np.all(lam < 1)
        assert np.all(np.diff(lam) > 0)          # later heads decay more slowly
        assert abs(lam[-1] - math.exp(-1.0 / 256.0)) < 1e-15   # the last head is always exp(-2^-8)


# --------------------------------------------------------------------------- three codings agree
@pytest.mark.parametrize("N", [1, 2, 3, 17, 64, 257])
def test_three_forms_agree(N):
    rng = np.random.default_rng(N)
    H, Dk, Dv = 2, 5, 3
    lam = rng.uniform(0.05, 1.0, H)
    lam[0] = 1.0 if N % 2 else lam[0]
    q, k, v = _rand(rng, N, H, Dk), _rand(rng, N, H, Dk), _rand(rng, N, H, Dv)
    s0 = _rand(rng, 1, H, Dk, Dv)
    o_r, s_r = oracle.prefill_recurrent(q, k, v, lam=lam, initial_state=s0, return_final_state=True)
    o_q, s_q = oracle.prefill_quadratic(q, k, v, lam=lam, initial_state=s0, return_final_state=True)
    _close(o_r, o_q, 1e-11)
    _close(s_r, s_q, 1e-11)
    if N <= 17:
        o_b, s_b = oracle.prefill_bruteforce(q, k, v, lam=lam, initial_state=s0, return_final_state=True)
        _close(o_r, o_b, 1e-12)
        _close(s_r, s_b, 1e-12)


def test_three_forms_agree_varlen_with_empty_sequences():
    rng = np.random.default_rng(7)
    lens = [3, 0, 5, 1, 0]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, H, Dk, Dv = int(cu[-1]), 3, 4, 4
    lam = oracle.decay(H)
    q, k, v = _rand(rng, T, H, Dk), _rand(rng, T, H, Dk), _rand(rng, T, H, Dv)
    s0 = _rand(rng, len(lens), H, Dk, Dv)
    outs = [f(q, k, v, cu_seqlens=cu, lam=lam, initial_state=s0, return_final_state=True) for f in ALL_FORMS]
    for o, s in outs[1:]:
        _close(outs[0][0], o)
        _close(outs[0][1], s)
    # an empty sequence passes its state through unchanged
    _close(outs[0][1][1], s0[1], 0.0)
    _close(outs[0][1][4], s0[4], 0.0)


# --------------------------------------------------------------------------- closed forms
def test_lambda_one_is_causal_cumulative_sum():
    """lambda = 1: o_t = q_t (sum_{s<=t} k_s^T v_s) = (tril(Q K^T) V)_t, computed with numpy.cumsum."""
    rng = np.random.default_rng(1)
    N, H, Dk, Dv = 40, 2, 6, 4
    q, k, v = _rand(rng, N, H, Dk), _rand(rng, N, H, Dk), _rand(rng, N, H, Dv)
    outer = np.einsum("thi,thj->thij", k, v)
    S = np.cumsum(outer, axis=0)
    want = np.einsum("thi,thij->thj", q, S)
    for form in (oracle.prefill_recurrent, oracle.prefill_quadratic):
        o, sN = form(q, k, v, lam=np.ones(H), return_final_state=True)
        _close(o, want, 1e-12)
        _close(sN[0], S[-1], 1e-12)


@pytest.mark.parametrize("lam", [0.3, 0.9, 0.999, 1.0])
def test_constant_inputs_geometric_series(lam):
    """q_t = q, k_t = k, v_t = v: o_t = (q.k) v (1 - lam^t)/(1 - lam) + lam^t q S0 (t = 1..N),
    and S_N = lam^N S0 + k^T v (1 - lam^N)/(1 - lam); for lam = 1 the geometric sum is t."""
    rng = np.random.default_rng(2)
    N, Dk, Dv = 50, 4, 3
    qv, kv, vv = _rand(rng, Dk), _rand(rng, Dk), _rand(rng, Dv)
    s0 = _rand(rng, Dk, Dv)
    q = np.broadcast_to(qv, (N, 1, Dk)).copy()
    k = np.broadcast_to(kv, (N, 1, Dk)).copy()
    v = np.broadcast_to(vv, (N, 1, Dv)).copy()
    t = np.arange(1, N + 1, dtype=np.float64)
    geo = t if lam == 1.0 else (1 - lam ** t) / (1 - lam)
    want = (qv @ kv) * geo[:, None] * vv[None, :] + (lam ** t)[:, None] * (qv @ s0)[None, :]
    geoN = N if lam == 1.0 else (1 - lam ** N) / (1 - lam)
    wantS = lam ** N * s0 + np.outer(kv, vv) * geoN
    for form in (oracle.prefill_recurrent, oracle.prefill_quadratic):
        o, sN = form(q, k, v, lam=[lam], initial_state=s0[None, None], return_final_state=True)
        _close(o[:, 0, :], want, 1e-12)
        _close(sN[0, 0], wantS, 1e-12)


def test_impulse_response():
    """One nonzero token s with k = e_a, v = e_b: o_t = lam^(t-s) q_t[a] e_b for t >= s and 0 before."""
    rng = np.random.default_rng(3)
    N, Dk, Dv, s, a, b, lam = 30, 5, 4, 11, 2, 3, 0.8
    q = _rand(rng, N, 1, Dk)
    k = np.zeros((N, 1, Dk))
    v = np.zeros((N, 1, Dv))
    k[s, 0, a] = 1.0
    v[s, 0, b] = 1.0
    want = np.zeros((N, 1, Dv))
    for t in range(s, N):
        want[t, 0, b] = lam ** (t - s) * q[t, 0, a]
    for form in (oracle.prefill_recurrent, oracle.prefill_quadratic):
        _close(form(q, k, v, lam=[lam]), want, 1e-14)


def test_single_token_and_zero_decay():
    rng = np.random.default_rng(4)
    Dk, Dv = 6, 5
    q, k, v = _rand(rng, 1, 1, Dk), _rand(rng, 1, 1, Dk), _rand(rng, 1, 1, Dv)
    s0 = _rand(rng, 1, 1, Dk, Dv)
    lam = 0.7
    want = lam * (q[0, 0] @ s0[0, 0]) + (q[0, 0] @ k[0, 0]) * v[0, 0]
    for form in ALL_FORMS:
        _close(form(q, k, v, lam=[lam], initial_state=s0)[0, 0], want, 1e-14)
    # lam = 0: only the current token survives, o_t = (q_t . k_t) v_t, initial state forgotten
    N = 9
    q, k, v = _rand(rng, N, 1, Dk), _rand(rng, N, 1, Dk), _rand(rng, N, 1, Dv)
    want = np.einsum("ti,ti->t", q[:, 0], k[:, 0])[:, None] * v[:, 0]
    for form in ALL_FORMS:
        _close(form(q, k, v, lam=[0.0], initial_state=_rand(rng, 1, 1, Dk, Dv))[:, 0], want, 1e-14)


# --------------------------------------------------------------------------- composition invariants
def test_split_with_state_handoff_equals_one_call():
    """Shard composition: run [0, N1) then [N1, N) from the first call's final state."""
    rng = np.random.default_rng(5)
    N, N1, H, D = 300, 137, 2, 8
    lam = oracle.decay(H)
    q, k, v = _rand(rng, N, H, D), _rand(rng, N, H, D), _rand(rng, N, H, D)
    s0 = _rand(rng, 1, H, D, D)
    o, sN = oracle.prefill_recurrent(q, k, v, lam=lam, initial_state=s0, return_final_state=True)
    o1, s1 = oracle.prefill_quadratic(q[:N1], k[:N1], v[:N1], lam=lam, initial_state=s0, return_final_state=True)
    o2, s2 = oracle.prefill_quadratic(q[N1:], k[N1:], v[N1:], lam=lam, initial_state=s1, return_final_state=True)
    _close(np.concatenate([o1, o2]), o, 1e-11)
    _close(s2, sN, 1e-11)


def test_local_recursion_plus_global_correction():
    """The shard reading of the context-parallel section: each shard from a zero state, then
    o_t += lambda^(t+1) q_t S_in (t local, 0-based) and S_out = lambda^L S_in + dS."""
    rng = np.random.default_rng(6)
    L, R, H, D = 40, 3, 2, 6
    lam = oracle.decay(H)
    N = L * R
    q, k, v = _rand(rng, N, H, D), _rand(rng, N, H, D), _rand(rng, N, H, D)
    want = oracle.prefill_recurrent(q, k, v, lam=lam)
    S_in = np.zeros((H, D, D))
    got = []
    t = np.arange(L)
    for r in range(R):
        sl = slice(r * L, (r + 1) * L)
        o_loc, dS = oracle.prefill_quadratic(q[sl], k[sl], v[sl], lam=lam, return_final_state=True)
        corr = np.stack([(lam[h] ** (t + 1))[:, None] * (q[sl, h] @ S_in[h]) for h in range(H)], axis=1)
        got.append(o_loc + corr)
        S_in = (lam ** L)[:, None, None] * S_in + dS[0]
    _close(np.concatenate(got), want, 1e-11)


def test_decode_steps_equal_prefill():
    rng = np.random.default_rng(8)
    B, N, H, D = 2, 12, 3, 4
    lam = oracle.decay(H)
    q, k, v = _rand(rng, B, N, H, D), _rand(rng, B, N, H, D), _rand(rng, B, N, H, D)
    s0 = _rand(rng, B, H, D, D)
    o, sN = oracle.prefill_quadratic(q, k, v, lam=lam, initial_state=s0, return_final_state=True)
    S = s0
    for t in range(N):
        ot, S = oracle.decode_step(q[:, t], k[:, t], v[:, t], S, lam=lam)
        _close(ot, o[:, t], 1e-12)
    _close(S, sN, 1e-12)


def test_varlen_equals_separate_calls():
    rng = np.random.default_rng(9)
    lens = [7, 1, 20, 4]
    cu = np.concatenate([[0], np.cumsum(lens)])
    H, D = 2, 5
    lam = oracle.decay(H)
    T = int(cu[-1])
    q, k, v = _rand(rng, T, H, D), _rand(rng, T, H, D), _rand(rng, T, H, D)
    s0 = _rand(rng, len(lens), H, D, D)
    o, sN = oracle.prefill_recurrent(q, k, v, cu_seqlens=cu, lam=lam, initial_state=s0, return_final_state=True)
    for i in range(len(lens)):
        sl = slice(int(cu[i]), int(cu[i + 1]))
        oi, si = oracle.prefill_quadratic(q[sl], k[sl], v[sl], lam=lam, initial_state=s0[i:i + 1],
                                          return_final_state=True)
        _close(o[sl], oi, 1e-12)
        _close(sN[i], si[0], 1e-12)


def test_value_column_split_and_linearity():
    rng = np.random.default_rng(10)
    N, H, Dk, Dv = 33, 2, 4, 6
    lam = oracle.decay(H)
    q, k = _rand(rng, N, H, Dk), _rand(rng, N, H, Dk)
    v1, v2 = _rand(rng, N, H, Dv), _rand(rng, N, H, Dv)
    s1, s2 = _rand(rng, 1, H, Dk, Dv), _rand(rng, 1, H, Dk, Dv)
    o, sN = oracle.prefill_recurrent(q, k, v1, lam=lam, initial_state=s1, return_final_state=True)
    # columns of v are independent problems
    oa, sa = oracle.prefill_recurrent(q, k, v1[..., :2], lam=lam, initial_state=s1[..., :2], return_final_state=True)
    ob, sb = oracle.prefill_recurrent(q, k, v1[..., 2:], lam=lam, initial_state=s1[..., 2:], return_final_state=True)
    _close(np.concatenate([oa, ob], -1), o, 0.0)
    _close(np.concatenate([sa, sb], -1), sN, 0.0)
    # linear in (v, S0) jointly
    a, b = 0.75, -1.5
    o12 = oracle.prefill_recurrent(q, k, a * v1 + b * v2, lam=lam, initial_state=a * s1 + b * s2)
    o2 = oracle.prefill_recurrent(q, k, v2, lam=lam, initial_state=s2)
    _close(o12, a * o + b * o2, 1e-12)


# --------------------------------------------------------------------------- planted mistakes
def _mutant(kind):
    """A copy of the quadratic form with one plausible mistake planted in it."""
    def f(q, k, v, lam, initial_state=None):
        q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
        N, H, _ = q.shape
        t = np.arange(N)
        d = (t[:, None] - t[None, :]).astype(float)
        out = np.zeros((N, H, v.shape[2]))
        for h in range(H):
            lh = lam[h]
            if kind == "exponent_off_by_one":
                M = np.where(d >= 0, lh ** (np.maximum(d, 0) + 1), 0.0)
            elif kind == "strict_causal_mask":
                M = np.where(d > 0, lh ** np.maximum(d, 0), 0.0)
            elif kind == "anticausal":
                M = np.where(d <= 0, lh ** np.maximum(-d, 0), 0.0)
            else:
                M = np.where(d >= 0, lh ** np.maximum(d, 0), 0.0)
            Q, K, V = q[:, h], k[:, h], v[:, h]
            out[:, h] = ((Q @ K.T) * M) @ V
            if initial_state is not None:
                S0 = initial_state[0, h]
                if kind == "state_not_decayed_first":
                    out[:, h] += (lh ** t)[:, None] * (Q @ S0)
                elif kind == "state_transposed":
                    out[:, h] += (lh ** (t + 1))[:, None] * (Q @ S0.T)
                elif kind == "state_dropped":
                    pass
                else:
                    out[:, h] += (lh ** (t + 1))[:, None] * (Q @ S0)
        return out
    return f


@pytest.mark.parametrize("kind", ["exponent_off_by_one", "strict_causal_mask", "anticausal",
                                  "state_not_decayed_first", "state_transposed", "state_dropped"])
def test_pins_catch_planted_mistakes(kind):
    """Each planted mistake must break the hand-worked examples or a closed form."""
    f = _mutant(kind)
    caught = False
    for case in _golden_cases()["cases"]:
        if case.get("cu_seqlens") is not None:
            continue
        q, k, v = (np.array(case[x], np.float64) for x in ("q", "k", "v"))
        s0 = None if case["initial_state"] is None else np.array(case["initial_state"])
        if not np.allclose(f(q, k, v, case["lam"], s0), np.array(case["o"]), rtol=0, atol=1e-12):
            caught = True
    # constant-input closed form with a non-symmetric initial state
    rng = np.random.default_rng(11)
    N, D, lam = 20, 3, 0.6
    qv, kv, vv = _rand(rng, D), _rand(rng, D), _rand(rng, D)
    s0 = _rand(rng, D, D)
    q = np.broadcast_to(qv, (N, 1, D)).copy()
    k = np.broadcast_to(kv, (N, 1, D)).copy()
    v = np.broadcast_to(vv, (N, 1, D)).copy()
    t = np.arange(1, N + 1)
    want = (qv @ kv) * ((1 - lam ** t) / (1 - lam))[:, None] * vv + (lam ** t)[:, None] * (qv @ s0)
    if not np.allclose(f(q, k, v, [lam], s0[None, None])[:, 0], want, rtol=0, atol=1e-12):
        caught = True
    assert caught, f"planted mistake {kind!r} was not caught by any pin"
    # and the unmutated coding passes the same checks
    assert np.allclose(_mutant("none")(q, k, v, [lam], s0[None, None])[:, 0], want, rtol=0, atol=1e-12)
