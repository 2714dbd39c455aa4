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
from linear_attention_hybrid_b200 import la_cp_entry_state, la_prefill, la_shard_state
from tests.parity_util import check

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")


def _oracle_state(k, v, lam):
    """The state from a zero start: the oracle's final state with no initial state."""
    q = np.zeros_like(k)
    _, s = oracle.prefill_recurrent(q, k, v, lam=lam, return_final_state=True)
    return s


@pytest.mark.parametrize("B, N, H", [(1, 4096, 4), (2, 1000, 3), (1, 128, 2), (1, 300, 16)])
def test_shard_state_matches_oracle(B, N, H):
    D = 128
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


@pytest.mark.parametrize("R, L, with_state", [(2, 2048, False), (4, 1024, True), (3, 1000, True), (8, 512, False)])
def test_context_parallel_equals_one_prefill(R, L, with_state):
    B, H, D = 2, 4, 128
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
