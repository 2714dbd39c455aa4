"""Context parallelism on one GPU: the R ranks of a context-parallel group emulated one after
another (each rank's steps are independent kernels; nothing waits on another rank), checked
against the oracle over the whole sequences. Per rank: la_shard_state (the shard's state from a
zero start), then, from every shard's state in rank order, la_cp_entry_state (the state entering
the shard) and la_prefill from it."""

import numpy as np
import pytest
import torch

import oracle
from linear_attention_hybrid_b200 import inputs as W
from linear_attention_hybrid_b200 import la_cp_entry_state, la_get_device_error, la_prefill, la_shard_state
from tests.parity_util import check

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


@pytest.fixture(autouse=True)
def _device_clean():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    assert la_get_device_error() == 0, "a kernel recorded a device-side status"


def _oracle_state(k, v, lam):
    """The state from a zero start: the oracle's final state with no initial state."""
    q = np.zeros_like(k)
    _, s = oracle.prefill_recurrent(q, k, v, lam=lam, return_final_state=True)
    return s


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("B, N, H", [(1, 4096, 4), (2, 1000, 3), (1, 128, 2), (1, 300, 16)])
def test_shard_state_matches_oracle(B, N, H, D):
    q, k, v = W.make_qkv((B, N), H, D, seed=N + H)
    ds = la_shard_state(k.to(DEV), v.to(DEV))
    torch.cuda.synchronize()
    want = _oracle_state(k.double().numpy(), v.double().numpy(), oracle.decay(H))
    check(ds.double().cpu().numpy(), want, torch.bfloat16, "delta_state")


def test_shard_state_empty_shard_is_zero():
    k = torch.zeros((2, 0, 3, 128), dtype=torch.bfloat16, device=DEV)
    ds = la_shard_state(k, k)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ds).item() == 0


def test_entry_state_rank0_is_initial_state():
    s0 = W.make_state((2,), 3, 128, 128, std=0.1, seed=5).to(DEV)
    g = torch.randn((4, 2, 3, 128, 128), device=DEV)
    s_in = la_cp_entry_state(g, 0, 512, initial_state=s0)
    torch.cuda.synchronize()
    assert torch.equal(s_in, s0)
    z = la_cp_entry_state(g, 0, 512)
    torch.cuda.synchronize()
    assert torch.count_nonzero(z).item() == 0


@pytest.mark.parametrize("R, L, with_state, D", [(2, 2048, False, 128), (4, 1024, True, 128), (3, 1000, True, 128),
                                                (8, 512, False, 128), (3, 1000, True, 64), (4, 1024, False, 64)])
def test_context_parallel_equals_one_prefill(R, L, with_state, D):
    B, H = 2, 4
    N = R * L
    q, k, v = W.make_qkv((B, N), H, D, seed=R * 7 + L)
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=R).to(DEV) if with_state else None
    qd, kd, vd = (x.to(DEV) for x in (q, k, v))
    shards = [(qd[:, r * L:(r + 1) * L].contiguous(), kd[:, r * L:(r + 1) * L].contiguous(),
               vd[:, r * L:(r + 1) * L].contiguous()) for r in range(R)]
    gathered = torch.stack([la_shard_state(ks, vs) for _, ks, vs in shards])
    outs, last_state = [], None
    for r, (qs, ks, vs) in enumerate(shards):
        s_in = la_cp_entry_state(gathered, r, L, initial_state=s0)
        o, sN = la_prefill(qs, ks, vs, initial_state=s_in, return_final_state=True, out_dtype=torch.float32)
        outs.append(o)
        last_state = sN
    torch.cuda.synchronize()
    got_o = torch.cat(outs, dim=1).double().cpu().numpy()
    want_o, want_s = oracle.prefill_recurrent(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                              lam=oracle.decay(H),
                                              initial_state=None if s0 is None else s0.double().cpu().numpy(),
                                              return_final_state=True)
    check(got_o, want_o, torch.bfloat16, "o")
    check(last_state.double().cpu().numpy(), want_s, torch.bfloat16, "final state")


# --------------------------------------------------------------------------- context-parallel backward
from linear_attention_hybrid_b200 import la_cp_reverse_entry_state, la_prefill_backward, la_shard_state_reverse  # noqa: E402


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("B, N, H", [(1, 4096, 4), (2, 1000, 3), (1, 128, 2), (1, 300, 16)])
def test_shard_state_reverse_matches_oracle(B, N, H, D):
    q, _, _ = W.make_qkv((B, N), H, D, seed=N + H)
    g = W.make_grad_out((B, N), H, D, seed=N + H + 1)
    dh = la_shard_state_reverse(q.to(DEV), g.to(DEV))
    torch.cuda.synchronize()
    z = np.zeros(tuple(q.shape))
    want = oracle.prefill_backward_recurrent(q.double().numpy(), z, z, g.double().numpy(), lam=oracle.decay(H))[3]
    check(dh.double().cpu().numpy(), want, torch.bfloat16, "reversed shard state")


def test_reverse_entry_state_last_rank_is_final_state_gradient():
    dsn = W.make_state((2,), 3, 128, 128, std=0.1, seed=5).to(DEV)
    g = torch.randn((4, 2, 3, 128, 128), device=DEV)
    h = la_cp_reverse_entry_state(g, 3, 512, d_final_state=dsn)
    torch.cuda.synchronize()
    assert torch.equal(h, dsn)


@pytest.mark.parametrize("R, L, D", [(2, 2048, 128), (3, 1000, 128), (4, 1024, 128), (3, 1000, 64)])
def test_context_parallel_backward_equals_one_backward(R, L, D):
    B, H = 2, 4
    N = R * L
    q, k, v = W.make_qkv((B, N), H, D, seed=R * 5 + L)
    g = W.make_grad_out((B, N), H, D, seed=R * 5 + L + 1)
    s0 = W.make_state((B,), H, D, D, std=0.1, seed=R)
    dsn = W.make_state((B,), H, D, D, std=0.1, seed=R + 1)
    qd, kd, vd, gd, s0d, dsnd = (x.to(DEV) for x in (q, k, v, g, s0, dsn))
    sl = [slice(r * L, (r + 1) * L) for r in range(R)]
    shard = lambda x, r: x[:, sl[r]].contiguous()  # noqa: E731
    fwd = torch.stack([la_shard_state(shard(kd, r), shard(vd, r)) for r in range(R)])
    rev = torch.stack([la_shard_state_reverse(shard(qd, r), shard(gd, r)) for r in range(R)])
    outs = []
    for r in range(R):
        s_in = la_cp_entry_state(fwd, r, L, initial_state=s0d)
        h_in = la_cp_reverse_entry_state(rev, r, L, d_final_state=dsnd)
        outs.append(la_prefill_backward(shard(qd, r), shard(kd, r), shard(vd, r), shard(gd, r), initial_state=s_in,
                                        d_final_state=h_in, return_d_initial_state=True, out_dtype=torch.float32))
    torch.cuda.synchronize()
    want = oracle.prefill_backward_recurrent(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                             g.double().numpy(), lam=oracle.decay(H), initial_state=s0.double().numpy(),
                                             d_final_state=dsn.double().numpy())
    for i, name in enumerate(("dq", "dk", "dv")):
        got = torch.cat([o[i] for o in outs], dim=1).double().cpu().numpy()
        check(got, want[i], torch.bfloat16, name)
    check(outs[0][3].double().cpu().numpy(), want[3], torch.bfloat16, "d_initial_state")


# --------------------------------------------------------------------------- context parallelism over varlen batches
from linear_attention_hybrid_b200.binding import (VarlenShard, varlen_cp_backward, varlen_cp_forward,  # noqa: E402
                                                  varlen_cp_send)


def _varlen_cp_batch(R, D, lengths, seed):
    H = 4
    T = sum(lengths)
    lengths = list(lengths)
    lengths[-1] += (-T) % R
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    T = int(cu[-1])
    q, k, v = W.make_qkv((T,), H, D, seed=seed)
    g = W.make_grad_out((T,), H, D, seed=seed + 1)
    nseq = len(lengths)
    s0 = W.make_state((nseq,), H, D, D, std=0.1, seed=seed + 2)
    dsn = W.make_state((nseq,), H, D, D, std=0.1, seed=seed + 3)
    return cu, H, (q, k, v, g), s0, dsn


# sequences crossing several shard boundaries, empty sequences (on a boundary and at the end), a boundary that
# falls between two sequences, and a shard inside one sequence
VARLEN_CP_CASES = [
    (2, 128, (1500, 700, 0, 1900, 0), 5),
    (3, 128, (333, 0, 2500, 41, 128, 1000, 0), 6),
    (4, 128, (1024, 0, 3000, 5, 1000, 0), 7),
    (8, 128, (4000, 3, 0, 900, 2600, 1, 0), 8),
    (3, 64, (700, 2000, 0, 333, 0), 9),
]


@pytest.mark.parametrize("R, D, lengths, seed", VARLEN_CP_CASES)
def test_varlen_context_parallel_equals_one_call(R, D, lengths, seed):
    """The R ranks of la_prefill_varlen_cp / la_prefill_varlen_cp_backward emulated one after another on one
    GPU (each rank's kernels are independent; the all-gather is a stack of their contributions): outputs,
    gradients, final states and initial-state gradients equal one oracle call over the whole packed batch."""
    cu, H, (q, k, v, g), s0, dsn = _varlen_cp_batch(R, D, lengths, seed)
    L = int(cu[-1]) // R
    qd, kd, vd, gd, s0d, dsnd = (x.to(DEV) for x in (q, k, v, g, s0, dsn))
    shards = [VarlenShard(cu, R, r) for r in range(R)]
    loc = [tuple(x[r * L:(r + 1) * L].contiguous() for x in (qd, kd, vd, gd)) for r in range(R)]
    fwd = torch.stack([varlen_cp_send(lk, lv, sh) for (lq, lk, lv, lg), sh in zip(loc, shards)])
    both = torch.stack([varlen_cp_send(lk, lv, sh, q=lq, dout=lg) for (lq, lk, lv, lg), sh in zip(loc, shards)])
    outs = [varlen_cp_forward(lq, lk, lv, sh, fwd, s0d, True, out_dtype=torch.float32)
            for (lq, lk, lv, lg), sh in zip(loc, shards)]
    grads = [varlen_cp_backward(lq, lk, lv, lg, sh, both, s0d, dsnd, out_dtype=torch.float32)
             for (lq, lk, lv, lg), sh in zip(loc, shards)]
    torch.cuda.synchronize()
    lam = oracle.decay(H)
    q64, k64, v64, g64 = (x.double().numpy() for x in (q, k, v, g))
    want_o, want_s = oracle.prefill_recurrent(q64, k64, v64, cu_seqlens=cu, lam=lam, initial_state=s0.double().numpy(),
                                              return_final_state=True)
    check(torch.cat([o for o, _, _ in outs]).double().cpu().numpy(), want_o, torch.bfloat16, "o")
    fin = {i: f for _, fs, ids in outs for i, f in zip(ids, fs)}
    assert sorted(fin) == list(range(len(cu) - 1))
    check(torch.stack([fin[i] for i in sorted(fin)]).double().cpu().numpy(), want_s, torch.bfloat16, "final states")
    want = oracle.prefill_backward_recurrent(q64, k64, v64, g64, cu_seqlens=cu, lam=lam,
                                             initial_state=s0.double().numpy(), d_final_state=dsn.double().numpy())
    for n, name in enumerate(("dq", "dk", "dv")):
        check(torch.cat([x[n] for x in grads]).double().cpu().numpy(), want[n], torch.bfloat16, name)
    dinit = {i: d for *_, ds, ids in grads for i, d in zip(ids, ds)}
    assert sorted(dinit) == list(range(len(cu) - 1))
    check(torch.stack([dinit[i] for i in sorted(dinit)]).double().cpu().numpy(), want[3], torch.bfloat16,
          "initial-state gradients")
