"""Pins for the oracle's output norm + gate (y = gamma * o / sqrt(mean(o^2) + eps) * sigmoid(z), one RMS
group per (token, head)): a hand-worked example, library routines (torch's rms_norm and sigmoid in fp64),
the invariants of a normalisation, and planted mistakes."""

import math

import numpy as np
import pytest
import torch

import oracle


def test_hand_worked_example():
    # one token, one head, D = 2: o = (3, 4), mean(o^2) = 12.5; gate (0, ln 3): sigmoid = (1/2, 3/4);
    # weight (2, 1); eps = 0  ->  y = (2 * 3 / sqrt(12.5) / 2, 4 / sqrt(12.5) * 3 / 4)
    o = np.array([[[3.0, 4.0]]])
    z = np.array([[[0.0, math.log(3.0)]]])
    w = np.array([[2.0, 1.0]])
    y = oracle.norm_gate(o, z, w, 0.0)
    want = np.array([[[3.0 / math.sqrt(12.5), 3.0 / math.sqrt(12.5)]]])
    np.testing.assert_allclose(y, want, rtol=1e-15, atol=0)


def test_matches_library_rms_norm_and_sigmoid():
    rng = np.random.default_rng(0)
    T, H, D, eps = 7, 3, 16, 1e-6
    o, z = rng.standard_normal((T, H, D)), rng.standard_normal((T, H, D))
    w = rng.standard_normal((H, D))
    got = oracle.norm_gate(o, z, w, eps)
    ot = torch.from_numpy(o)
    want = torch.stack([torch.nn.functional.rms_norm(ot[:, h], (D,), weight=torch.from_numpy(w[h]), eps=eps)
                        for h in range(H)], dim=1) * torch.sigmoid(torch.from_numpy(z))
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-13, atol=1e-14)


def test_normalisation_invariants():
    rng = np.random.default_rng(1)
    T, H, D = 5, 2, 8
    o = rng.standard_normal((T, H, D))
    ones = np.ones((H, D))
    big = np.full((T, H, D), 60.0)          # sigmoid = 1 to fp64 precision
    y = oracle.norm_gate(o, big, ones, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)   # unit RMS per group
    scaled = oracle.norm_gate(o * np.array([2.5, 1e-3, 7.0, 1.0, 40.0])[:, None, None], big, ones, 0.0)
    np.testing.assert_allclose(scaled, y, rtol=1e-13)                                 # per-group scale invariance
    zero = oracle.norm_gate(o, np.zeros_like(o), ones, 0.0)
    np.testing.assert_allclose(zero, 0.5 * y, rtol=1e-15)                             # sigmoid(0) = 1/2
    # groups are the heads: changing head 1 leaves head 0's output alone
    o2 = o.copy()
    o2[:, 1] *= 3.0
    o2[:, 1, 0] += 1.0
    np.testing.assert_array_equal(oracle.norm_gate(o2, big, ones, 0.0)[:, 0], y[:, 0])


def test_eps_keeps_zero_rows_finite():
    y = oracle.norm_gate(np.zeros((2, 1, 4)), np.zeros((2, 1, 4)), np.ones((1, 4)), 1e-6)
    assert np.all(y == 0)


def _mutant(kind):
    def f(o, z, w, eps):
        if kind == "norm_over_all_heads":
            ms = np.mean(o * o, axis=(-2, -1), keepdims=True)
        elif kind == "sum_not_mean":
            ms = np.sum(o * o, axis=-1, keepdims=True)
        else:
            ms = np.mean(o * o, axis=-1, keepdims=True)
        g = 1.0 / (1.0 + np.exp(z)) if kind == "gate_sign" else 1.0 / (1.0 + np.exp(-z))
        if kind == "eps_outside_sqrt":
            return w * o / (np.sqrt(ms) + eps) * g
        return w * o / np.sqrt(ms + eps) * g
    return f


@pytest.mark.parametrize("kind", ["norm_over_all_heads", "sum_not_mean", "gate_sign", "eps_outside_sqrt"])
def test_pins_catch_planted_mistakes(kind):
    rng = np.random.default_rng(2)
    T, H, D, eps = 6, 3, 16, 0.5
    o, z, w = rng.standard_normal((T, H, D)), rng.standard_normal((T, H, D)), rng.standard_normal((H, D))
    ot = torch.from_numpy(o)
    lib = torch.stack([torch.nn.functional.rms_norm(ot[:, h], (D,), weight=torch.from_numpy(w[h]), eps=eps)
                       for h in range(H)], dim=1) * torch.sigmoid(torch.from_numpy(z))
    assert not np.allclose(_mutant(kind)(o, z, w, eps), lib.numpy(), rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(_mutant("none")(o, z, w, eps), lib.numpy(), rtol=1e-13, atol=1e-14)
