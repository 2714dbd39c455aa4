"""Lightning Attention oracle: plain, slow, obviously correct fp64 CPU code.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or run anything here. The CUDA
library never imports this package and this package never imports the CUDA
library; the two share no code (the seeded input generator, which holds none
of the operator's arithmetic, is the only module both sides are fed from).

Source of the operator (Ling & Ring 2.6 Technical Report, blog post at
news.neo-ai.one/en/article/3021):
  * section "Hybrid Linear Attention": Lightning Attention is the linear layer
    of the hybrid stack and brings the sequence cost from O(n^2) to O(n);
  * section "Long-Context Training: Context Parallel for Lightning Attention":
    the layer carries a state recursively along the sequence, and shards can
    be computed locally and corrected with the states of earlier shards.
The pages print no formula. The specified operator is

    o_t = sum_{s<=t} lambda_h^(t-s) (q_t . k_s) v_s,  lambda_h = exp(-2^(-8(h+1)/H)),

with the state form S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t (S is
Dk x Dv, S[i, j] pairs k_i with v_j). Readings of points the pages leave open
(all listed in the design notes): the initial state decays once before the
first token; token t is included in o_t; h is 0-based; no 1/sqrt(D) scale,
normaliser, feature map or gate is applied inside the operator.

Three independent codings of that one definition:
  * ``prefill_recurrent`` -- the state recursion, in C (``la_oracle.c``),
    threaded over (sequence, head); also the timed CPU baseline;
  * ``prefill_quadratic`` -- the masked-decay matrix form
    O = ((Q K^T) * M) V + diag(lambda^(t+1)) Q S0, M[t, s] = lambda^(t-s) [s <= t],
    in numpy;
  * ``prefill_bruteforce`` -- the literal sums in plain Python loops (tiny
    inputs only).
``decode_step`` is one step of the recursion, in C.

The backward pass (the pages do not treat it) is the derivative of that
definition for a loss with gradients dO (of the outputs) and dS_N (of the final
state), in the same three codings: ``prefill_backward_recurrent`` (the adjoint
recursion, C), ``prefill_backward_quadratic`` (the matrix form, numpy) and
``prefill_backward_bruteforce`` (the literal sums).

Pins that tie these to something other than themselves (closed forms,
invariants, hand-worked examples) are in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libla_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile la_oracle.c into oracle/libla_oracle.so with gcc (fp64, -O2, pthreads)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", _LIB_PATH, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        dp = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.la_oracle_decay.argtypes = [ctypes.c_int, dp]
        lib.la_oracle_default_threads.argtypes = []
        lib.la_oracle_prefill_recurrent.argtypes = [dp, dp, dp, dp, i64p, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int, ctypes.c_int, dp, dp, dp, ctypes.c_int]
        lib.la_oracle_decode_step.argtypes = [dp, dp, dp, dp, dp, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int, ctypes.c_int, dp]
        lib.la_oracle_prefill_backward_recurrent.argtypes = [dp, dp, dp, dp, dp, dp, dp, i64p, ctypes.c_int,
                                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, dp, dp,
                                                             dp, ctypes.c_int]
        _lib = lib
    return _lib


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(a):
    """Widen to a C-contiguous float64 numpy array (exact for bf16 / fp32 inputs)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        import torch
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def default_threads() -> int:
    """CPUs in this process's affinity mask (what the threaded recurrence uses)."""
    return int(_load().la_oracle_default_threads())


def decay(H: int) -> np.ndarray:
    """lambda_h = exp(-2^(-8(h+1)/H)) for h = 0..H-1, in fp64."""
    lam = np.empty(H, dtype=np.float64)
    if _load().la_oracle_decay(H, _ptr(lam)) != 0:
        raise ValueError("H must be >= 1")
    return lam


def _packed(q, k, v, cu_seqlens, initial_state):
    """Accept [B, N, H, D] (uniform lengths) or packed [T, H, D] + cu_seqlens."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim == 4:
        B, N, H, Dk = q.shape
        Dv = v.shape[3]
        cu = np.arange(B + 1, dtype=np.int64) * N
        q, k, v = q.reshape(B * N, H, Dk), k.reshape(B * N, H, Dk), v.reshape(B * N, H, Dv)
        shape4 = (B, N)
    else:
        if cu_seqlens is None:
            cu = np.array([0, q.shape[0]], dtype=np.int64)
        else:
            cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
        shape4 = None
    T, H, Dk = q.shape
    Dv = v.shape[2]
    if k.shape != (T, H, Dk) or v.shape[:2] != (T, H) or int(cu[-1]) != T or int(cu[0]) != 0:
        raise ValueError("inconsistent shapes / cu_seqlens")
    s0 = _f64(initial_state)
    nseq = len(cu) - 1
    if s0 is not None:
        s0 = s0.reshape(nseq, H, Dk, Dv)
    return q, k, v, cu, s0, shape4


def _lam(H, lam):
    return decay(H) if lam is None else np.ascontiguousarray(np.broadcast_to(np.asarray(lam, np.float64), (H,)))


def prefill_recurrent(q, k, v, cu_seqlens=None, lam=None, initial_state=None, return_final_state=False,
                      nthreads: int = 0):
    """State recursion (C, fp64). Returns o (same leading shape as q) and optionally the final state."""
    q, k, v, cu, s0, shape4 = _packed(q, k, v, cu_seqlens, initial_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    nseq = len(cu) - 1
    lamv = _lam(H, lam)
    o = np.empty((T, H, Dv), dtype=np.float64)
    sN = np.empty((nseq, H, Dk, Dv), dtype=np.float64) if return_final_state else None
    rc = _load().la_oracle_prefill_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                             cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), nseq, H, Dk, Dv,
                                             _ptr(lamv), _ptr(s0), _ptr(sN), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"la_oracle_prefill_recurrent failed ({rc})")
    if shape4 is not None:
        o = o.reshape(shape4[0], shape4[1], H, Dv)
    return (o, sN) if return_final_state else o


def prefill_quadratic(q, k, v, cu_seqlens=None, lam=None, initial_state=None, return_final_state=False):
    """Masked-decay matrix form (numpy, fp64), per sequence and head:
    O = ((Q K^T) * M) V + diag(lambda^(t+1)) Q S0 with M[t, s] = lambda^(t-s) for s <= t, else 0;
    final state lambda^n S0 + sum_s lambda^(n-1-s) k_s^T v_s (t, s 0-based)."""
    q, k, v, cu, s0, shape4 = _packed(q, k, v, cu_seqlens, initial_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    nseq = len(cu) - 1
    lamv = _lam(H, lam)
    o = np.zeros((T, H, Dv), dtype=np.float64)
    sN = np.zeros((nseq, H, Dk, Dv), dtype=np.float64)
    for i in range(nseq):
        a, b = int(cu[i]), int(cu[i + 1])
        n = b - a
        t = np.arange(n)
        diff = (t[:, None] - t[None, :]).astype(np.float64)
        for h in range(H):
            Q, K, V = q[a:b, h, :], k[a:b, h, :], v[a:b, h, :]
            lh = lamv[h]
            M = np.where(diff >= 0, np.power(lh, np.maximum(diff, 0.0)), 0.0)
            out = ((Q @ K.T) * M) @ V
            w = np.power(lh, (n - 1 - t).astype(np.float64))   # lambda^(n-1-s)
            S = (K * w[:, None]).T @ V
            if s0 is not None:
                out = out + np.power(lh, (t + 1).astype(np.float64))[:, None] * (Q @ s0[i, h])
                S = S + lh ** n * s0[i, h]
            o[a:b, h, :] = out
            sN[i, h] = S
    if shape4 is not None:
        o = o.reshape(shape4[0], shape4[1], H, Dv)
    return (o, sN) if return_final_state else o


def prefill_bruteforce(q, k, v, cu_seqlens=None, lam=None, initial_state=None, return_final_state=False):
    """The literal sums of the definition in plain Python loops (tiny inputs only):
    o_t[j] = sum_{s<=t} sum_i lambda^(t-s) q_t[i] k_s[i] v_s[j] + sum_i lambda^(t+1) q_t[i] S0[i][j]."""
    q, k, v, cu, s0, shape4 = _packed(q, k, v, cu_seqlens, initial_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    if T > 64:
        raise ValueError("brute force is for tiny inputs")
    nseq = len(cu) - 1
    lamv = _lam(H, lam)
    o = np.zeros((T, H, Dv), dtype=np.float64)
    sN = np.zeros((nseq, H, Dk, Dv), dtype=np.float64)
    for sq in range(nseq):
        a, b = int(cu[sq]), int(cu[sq + 1])
        for h in range(H):
            lh = float(lamv[h])
            for t in range(b - a):
                for j in range(Dv):
                    acc = 0.0
                    for s in range(t + 1):
                        for i in range(Dk):
                            acc += lh ** (t - s) * q[a + t, h, i] * k[a + s, h, i] * v[a + s, h, j]
                    if s0 is not None:
                        for i in range(Dk):
                            acc += lh ** (t + 1) * q[a + t, h, i] * s0[sq, h, i, j]
                    o[a + t, h, j] = acc
            n = b - a
            for i in range(Dk):
                for j in range(Dv):
                    acc = 0.0 if s0 is None else lh ** n * s0[sq, h, i, j]
                    for s in range(n):
                        acc += lh ** (n - 1 - s) * k[a + s, h, i] * v[a + s, h, j]
                    sN[sq, h, i, j] = acc
    if shape4 is not None:
        o = o.reshape(shape4[0], shape4[1], H, Dv)
    return (o, sN) if return_final_state else o


def decode_step(q, k, v, state, lam=None):
    """One recurrent step (C, fp64): S <- lambda S + k^T v; o = q S. q, k: [B, H, Dk]; v: [B, H, Dv];
    state [B, H, Dk, Dv]. Returns (o, new_state); the input state is not modified."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    S = _f64(state).copy()
    B, H, Dk = q.shape
    Dv = v.shape[2]
    lamv = _lam(H, lam)
    o = np.empty((B, H, Dv), dtype=np.float64)
    rc = _load().la_oracle_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(S), B, H, Dk, Dv, _ptr(lamv))
    if rc != 0:
        raise RuntimeError("la_oracle_decode_step failed")
    return o, S



# --------------------------------------------------------------------------- backward pass
# The pages do not treat the backward pass. These are the gradients of the operator above for a loss
# L with dL/do_t = dO_t and dL/dS_N = dS_N (zero when absent): the derivative of the definition, in
# the same three codings as the forward.

def _packed_bwd(q, k, v, dout, cu_seqlens, initial_state, d_final_state):
    q, k, v, cu, s0, shape4 = _packed(q, k, v, cu_seqlens, initial_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    g = _f64(dout).reshape(T, H, Dv)
    dsN = _f64(d_final_state)
    if dsN is not None:
        dsN = dsN.reshape(len(cu) - 1, H, Dk, Dv)
    return q, k, v, g, cu, s0, dsN, shape4


def _unpack_bwd(dq, dk, dv, shape4):
    if shape4 is not None:
        B, N = shape4
        dq, dk, dv = (x.reshape(B, N, *x.shape[1:]) for x in (dq, dk, dv))
    return dq, dk, dv


def prefill_backward_recurrent(q, k, v, dout, cu_seqlens=None, lam=None, initial_state=None, d_final_state=None,
                               nthreads: int = 0):
    """Adjoint of the state recursion (C, fp64): a forward sweep gives dq_t = S_t dO_t, a reverse sweep
    G_t = q_t^T dO_t + lambda G_{t+1} (G starting from dS_N) gives dk_t = G_t v_t, dv_t = k_t G_t and
    dS_0 = lambda G_0. Returns (dq, dk, dv, dS_0) with dq, dk, dv shaped like q, k, v."""
    q, k, v, g, cu, s0, dsN, shape4 = _packed_bwd(q, k, v, dout, cu_seqlens, initial_state, d_final_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    nseq = len(cu) - 1
    lamv = _lam(H, lam)
    dq, dk, dv = np.empty((T, H, Dk)), np.empty((T, H, Dk)), np.empty((T, H, Dv))
    ds0 = np.empty((nseq, H, Dk, Dv))
    rc = _load().la_oracle_prefill_backward_recurrent(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dq), _ptr(dk), _ptr(dv),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), nseq, H, Dk, Dv, _ptr(lamv), _ptr(s0), _ptr(dsN),
        _ptr(ds0), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"la_oracle_prefill_backward_recurrent failed ({rc})")
    return (*_unpack_bwd(dq, dk, dv, shape4), ds0)


def prefill_backward_quadratic(q, k, v, dout, cu_seqlens=None, lam=None, initial_state=None, d_final_state=None):
    """Gradients of the masked-decay matrix form (numpy, fp64), per sequence and head, with
    M[t, s] = lambda^(t-s) [s <= t], E = (dO V^T) * M, w_t = lambda^(t+1), u_s = lambda^(n-1-s):
    dQ = E K + diag(w) dO S0^T;  dK = E^T Q + diag(u) V dS_N^T;  dV = ((Q K^T) * M)^T dO + diag(u) K dS_N;
    dS_0 = lambda^n dS_N + Q^T diag(w) dO."""
    q, k, v, g, cu, s0, dsN, shape4 = _packed_bwd(q, k, v, dout, cu_seqlens, initial_state, d_final_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    nseq = len(cu) - 1
    lamv = _lam(H, lam)
    dq, dk, dv = np.zeros((T, H, Dk)), np.zeros((T, H, Dk)), np.zeros((T, H, Dv))
    ds0 = np.zeros((nseq, H, Dk, Dv))
    for i in range(nseq):
        a, b = int(cu[i]), int(cu[i + 1])
        n = b - a
        t = np.arange(n)
        diff = (t[:, None] - t[None, :]).astype(np.float64)
        for h in range(H):
            Q, K, V, G = q[a:b, h], k[a:b, h], v[a:b, h], g[a:b, h]
            lh = lamv[h]
            M = np.where(diff >= 0, np.power(lh, np.maximum(diff, 0.0)), 0.0)
            E = (G @ V.T) * M
            w = np.power(lh, (t + 1).astype(np.float64))
            u = np.power(lh, (n - 1 - t).astype(np.float64))
            DQ, DK, DV = E @ K, E.T @ Q, ((Q @ K.T) * M).T @ G
            DS0 = Q.T @ (w[:, None] * G)
            if s0 is not None:
                DQ = DQ + w[:, None] * (G @ s0[i, h].T)
            if dsN is not None:
                DK = DK + u[:, None] * (V @ dsN[i, h].T)
                DV = DV + u[:, None] * (K @ dsN[i, h])
                DS0 = DS0 + lh ** n * dsN[i, h]
            dq[a:b, h], dk[a:b, h], dv[a:b, h], ds0[i, h] = DQ, DK, DV, DS0
    return (*_unpack_bwd(dq, dk, dv, shape4), ds0)


def prefill_backward_bruteforce(q, k, v, dout, cu_seqlens=None, lam=None, initial_state=None, d_final_state=None):
    """The gradients as literal sums in plain Python loops (tiny inputs only):
    dq_t[i] = sum_{s<=t} lambda^(t-s) k_s[i] (v_s . dO_t) + lambda^(t+1) sum_j S0[i][j] dO_t[j];
    dk_s[i] = sum_{t>=s} lambda^(t-s) q_t[i] (v_s . dO_t) + lambda^(n-1-s) sum_j dS_N[i][j] v_s[j];
    dv_s[j] = sum_{t>=s} lambda^(t-s) (q_t . k_s) dO_t[j] + lambda^(n-1-s) sum_i k_s[i] dS_N[i][j];
    dS_0[i][j] = lambda^n dS_N[i][j] + sum_t lambda^(t+1) q_t[i] dO_t[j]."""
    q, k, v, g, cu, s0, dsN, shape4 = _packed_bwd(q, k, v, dout, cu_seqlens, initial_state, d_final_state)
    T, H, Dk = q.shape
    Dv = v.shape[2]
    if T > 48:
        raise ValueError("brute force is for tiny inputs")
    nseq = len(cu) - 1
    lamv = _lam(H, lam)
    dq, dk, dv = np.zeros((T, H, Dk)), np.zeros((T, H, Dk)), np.zeros((T, H, Dv))
    ds0 = np.zeros((nseq, H, Dk, Dv))

    def dot(x, y):
        return sum(x[m] * y[m] for m in range(len(x)))

    for sq in range(nseq):
        a, b = int(cu[sq]), int(cu[sq + 1])
        n = b - a
        for h in range(H):
            lh = float(lamv[h])
            for t in range(n):
                for i in range(Dk):
                    acc = 0.0
                    for s in range(t + 1):
                        acc += lh ** (t - s) * k[a + s, h, i] * dot(v[a + s, h], g[a + t, h])
                    if s0 is not None:
                        acc += lh ** (t + 1) * sum(s0[sq, h, i, j] * g[a + t, h, j] for j in range(Dv))
                    dq[a + t, h, i] = acc
            for s in range(n):
                for i in range(Dk):
                    acc = 0.0
                    for t in range(s, n):
                        acc += lh ** (t - s) * q[a + t, h, i] * dot(v[a + s, h], g[a + t, h])
                    if dsN is not None:
                        acc += lh ** (n - 1 - s) * sum(dsN[sq, h, i, j] * v[a + s, h, j] for j in range(Dv))
                    dk[a + s, h, i] = acc
                for j in range(Dv):
                    acc = 0.0
                    for t in range(s, n):
                        acc += lh ** (t - s) * dot(q[a + t, h], k[a + s, h]) * g[a + t, h, j]
                    if dsN is not None:
                        acc += lh ** (n - 1 - s) * sum(k[a + s, h, i] * dsN[sq, h, i, j] for i in range(Dk))
                    dv[a + s, h, j] = acc
            for i in range(Dk):
                for j in range(Dv):
                    acc = 0.0 if dsN is None else lh ** n * dsN[sq, h, i, j]
                    for t in range(n):
                        acc += lh ** (t + 1) * q[a + t, h, i] * g[a + t, h, j]
                    ds0[sq, h, i, j] = acc
    return (*_unpack_bwd(dq, dk, dv, shape4), ds0)


# --------------------------------------------------------------------------- output norm + gate
# The report's "linghe" section names a fused "Group RMSNorm + Sigmoid Gate" among the BF16-inference
# fusions of the attention module, with no formula. Reading: each (token, head) output vector of D
# channels is one RMS group, scaled by a learned weight gamma[h, :] and gated elementwise by the sigmoid
# of a gate pre-activation z of the same shape as o (projected from the layer input outside the
# operator):  y = gamma * o / sqrt(mean_d(o^2) + eps) * sigmoid(z).

def norm_gate(o, gate, weight, eps):
    """y = weight[h] * o / sqrt(mean over the head's D channels of o^2 + eps) * sigmoid(gate), fp64.
    o, gate: [..., H, D]; weight: [H, D]."""
    o, z, w = _f64(o), _f64(gate), _f64(weight)
    ms = np.mean(o * o, axis=-1, keepdims=True)
    return w * o / np.sqrt(ms + float(eps)) * (1.0 / (1.0 + np.exp(-z)))


def prefill_norm_gate(q, k, v, gate, weight, eps, cu_seqlens=None, lam=None, initial_state=None,
                      return_final_state=False):
    """The operator (recurrent form) followed by norm_gate on its output."""
    r = prefill_recurrent(q, k, v, cu_seqlens=cu_seqlens, lam=lam, initial_state=initial_state,
                          return_final_state=return_final_state)
    o, sN = (r if return_final_state else (r, None))
    y = norm_gate(o, np.asarray(_f64(gate)).reshape(o.shape), weight, eps)
    return (y, sN) if return_final_state else y
