"""The multi-GPU path of ``bench.py`` on CPU: two ``gloo`` ranks (world size 2).

Prefill shards with no exchange on the data path: every rank runs its own seeded
batch of independent sequences and heads (weak scaling) and the job's time is the
slowest rank's. These tests run the same helpers ``bench.py`` uses under
``torch.distributed.run`` -- per-rank seeding, the max-over-ranks reduction and the
whole-job throughput -- on two processes, and check with the oracle that the
per-rank results are exactly the results of one batch holding both shards, i.e.
that sharding the batch needs no collective.
"""

import os
import socket
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

B, N, H, D = 1, 48, 2, 16


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import oracle
        from linear_attention_hybrid_b200 import inputs as W

        q, k, v = W.make_qkv((B, N), H, D, seed=bench.rank_seed(0, rank))
        o, s = oracle.prefill_recurrent(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                        lam=oracle.decay(H), return_final_state=True)
        ms = bench.max_over_ranks(1.0 + rank, world, torch.device("cpu"))
        got_q = [torch.zeros_like(q) for _ in range(world)]
        got_o = [torch.zeros(o.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(got_q, q)
        dist.all_gather(got_o, torch.from_numpy(np.ascontiguousarray(o)))
        np.save(os.path.join(out_dir, f"ms{rank}.npy"), np.array([ms]))
        if rank == 0:
            np.save(os.path.join(out_dir, "q.npy"), torch.stack(got_q).float().numpy())
            np.save(os.path.join(out_dir, "o.npy"), torch.stack(got_o).numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_ranks(tmp_path_factory):
    import oracle
    oracle.build()
    out = str(tmp_path_factory.mktemp("ranks"))
    mp.start_processes(_rank_main, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    return out


def test_slowest_rank_time_reaches_every_rank(two_ranks):
    for r in range(2):
        assert float(np.load(os.path.join(two_ranks, f"ms{r}.npy"))[0]) == 2.0


def test_ranks_get_distinct_batches(two_ranks):
    q = np.load(os.path.join(two_ranks, "q.npy"))
    assert q.shape == (2, B, N, H, D)
    assert not np.array_equal(q[0], q[1])


def test_shards_equal_one_batch_holding_both(two_ranks):
    """Per-rank outputs are bit-for-bit the oracle's output on the concatenated batch."""
    import bench
    import oracle
    from linear_attention_hybrid_b200 import inputs as W

    parts = [W.make_qkv((B, N), H, D, seed=bench.rank_seed(0, r)) for r in range(2)]
    q, k, v = (torch.cat([p[i] for p in parts], dim=0).double().numpy() for i in range(3))
    whole = oracle.prefill_recurrent(q, k, v, lam=oracle.decay(H))
    per_rank = np.load(os.path.join(two_ranks, "o.npy"))
    np.testing.assert_array_equal(per_rank.reshape(whole.shape), whole)


def test_weak_scaling_value():
    import bench
    assert bench.weak_scaling_value(1, 1000, 2.0) == pytest.approx(5e5)
    # two ranks, each 1000 units, slowest 2 ms: 2000 units in 2 ms
    assert bench.weak_scaling_value(2, 1000, 2.0) == pytest.approx(1e6)


def test_head_dim_option_names_the_workload():
    """--head-dim runs a specified workload's shape at the other head dimension under its own name, so
    nothing recorded for the specified workload (the chunk kernel's traffic record) is applied to it."""
    import argparse
    import bench
    from linear_attention_hybrid_b200 import inputs as W
    base = W.workloads()["prefill_b4_n4096"]
    same = bench.pick_workload(W, argparse.Namespace(workload="prefill_b4_n4096", head_dim=None))
    assert same == base
    assert bench.pick_workload(W, argparse.Namespace(workload="prefill_b4_n4096", head_dim=128)) == base
    d64 = bench.pick_workload(W, argparse.Namespace(workload="prefill_b4_n4096", head_dim=64))
    assert (d64.name, d64.D) == ("prefill_b4_n4096_d64", 64)
    assert (d64.B, d64.N, d64.H, d64.dtype) == (base.B, base.N, base.H, base.dtype)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    """Under torchrun only rank 0 times the oracle and prints; the other ranks exit 0 at once."""
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="prefill_b4_n4096", steps=1, warmup=0, gpus=2)
    assert bench.reference_arm(args) == 0


# --------------------------------------------------------------------------- context parallelism
# la_prefill_cp over two gloo ranks, with the per-rank steps done by the oracle (a test-only stand-in
# for the library's kernels, which need a GPU): checks the orchestration -- the shard states gathered in
# rank order, each rank's entry state, the last rank's final state -- against one oracle prefill over
# the whole sequences.
CP_B, CP_L, CP_H, CP_D = 2, 40, 3, 8


class _OracleShardOps:
    @staticmethod
    def shard_state(k, v, slopes):
        import oracle
        q = np.zeros(tuple(k.shape))
        _, s = oracle.prefill_recurrent(q, k.numpy(), v.numpy(), lam=oracle.decay(CP_H), return_final_state=True)
        return torch.from_numpy(s)

    @staticmethod
    def entry_state(gathered, rank, L, initial_state, slopes):
        import oracle
        lam = oracle.decay(CP_H)[None, :, None, None]
        s = np.zeros(tuple(gathered.shape[1:])) if initial_state is None else lam ** (rank * L) * initial_state.numpy()
        for rp in range(rank):
            s = s + lam ** ((rank - 1 - rp) * L) * gathered[rp].numpy()
        return torch.from_numpy(s)

    @staticmethod
    def prefill(q, k, v, s_in, return_final_state, slopes, out_dtype):
        import oracle
        o, s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), lam=oracle.decay(CP_H),
                                        initial_state=s_in.numpy(), return_final_state=True)
        return torch.from_numpy(o), torch.from_numpy(s)


def _cp_inputs(world):
    from linear_attention_hybrid_b200 import inputs as W
    q, k, v = W.make_qkv((CP_B, world * CP_L), CP_H, CP_D, seed=11)
    s0 = W.make_state((CP_B,), CP_H, CP_D, CP_D, std=0.1, seed=12)
    return [x.double() for x in (q, k, v)], s0.double()


def _cp_rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from linear_attention_hybrid_b200.binding import la_prefill_cp
        (q, k, v), s0 = _cp_inputs(world)
        sl = slice(rank * CP_L, (rank + 1) * CP_L)
        o, s = la_prefill_cp(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), initial_state=s0,
                             return_final_state=True, ops=_OracleShardOps)
        np.save(os.path.join(out_dir, f"cp_o{rank}.npy"), o.numpy())
        np.save(os.path.join(out_dir, f"cp_s{rank}.npy"), s.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_context_parallel_orchestration_equals_one_prefill(tmp_path):
    import oracle
    oracle.build()
    world = 2
    mp.start_processes(_cp_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    (q, k, v), s0 = _cp_inputs(world)
    want_o, want_s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), lam=oracle.decay(CP_H),
                                              initial_state=s0.numpy(), return_final_state=True)
    got_o = np.concatenate([np.load(os.path.join(tmp_path, f"cp_o{r}.npy")) for r in range(world)], axis=1)
    np.testing.assert_allclose(got_o, want_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(np.load(os.path.join(tmp_path, f"cp_s{world - 1}.npy")), want_s, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------- context-parallel backward
class _OracleBackwardOps(_OracleShardOps):
    @staticmethod
    def shard_state_reverse(q, dout, slopes):
        import oracle
        z = np.zeros(tuple(q.shape))
        return torch.from_numpy(oracle.prefill_backward_recurrent(q.numpy(), z, z, dout.numpy(),
                                                                  lam=oracle.decay(CP_H))[3])

    @staticmethod
    def reverse_entry_state(gathered, rank, L, d_final_state, slopes):
        import oracle
        lam = oracle.decay(CP_H)[None, :, None, None]
        R = gathered.shape[0]
        h = np.zeros(tuple(gathered.shape[1:])) if d_final_state is None else \
            lam ** ((R - 1 - rank) * L) * d_final_state.numpy()
        for rp in range(rank + 1, R):
            h = h + lam ** ((rp - rank - 1) * L) * gathered[rp].numpy()
        return torch.from_numpy(h)

    @staticmethod
    def backward(q, k, v, dout, s_in, h_in, slopes, out_dtype):
        import oracle
        return tuple(torch.from_numpy(x) for x in oracle.prefill_backward_recurrent(
            q.numpy(), k.numpy(), v.numpy(), dout.numpy(), lam=oracle.decay(CP_H), initial_state=s_in.numpy(),
            d_final_state=h_in.numpy()))


def _cp_bwd_inputs(world):
    (q, k, v), s0 = _cp_inputs(world)
    from linear_attention_hybrid_b200 import inputs as W
    g = W.make_grad_out((CP_B, world * CP_L), CP_H, CP_D, seed=13).double()
    dsn = W.make_state((CP_B,), CP_H, CP_D, CP_D, std=0.1, seed=14).double()
    return (q, k, v, g), s0, dsn


def _cp_bwd_rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from linear_attention_hybrid_b200.binding import la_prefill_cp_backward
        (q, k, v, g), s0, dsn = _cp_bwd_inputs(world)
        sl = slice(rank * CP_L, (rank + 1) * CP_L)
        grads = la_prefill_cp_backward(*(x[:, sl].contiguous() for x in (q, k, v, g)), initial_state=s0,
                                       d_final_state=dsn, ops=_OracleBackwardOps)
        for name, x in zip(("dq", "dk", "dv", "ds0"), grads):
            np.save(os.path.join(out_dir, f"cpb_{name}{rank}.npy"), x.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_context_parallel_backward_orchestration_equals_one_backward(tmp_path):
    import oracle
    oracle.build()
    world = 2
    mp.start_processes(_cp_bwd_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    (q, k, v, g), s0, dsn = _cp_bwd_inputs(world)
    want = oracle.prefill_backward_recurrent(q.numpy(), k.numpy(), v.numpy(), g.numpy(), lam=oracle.decay(CP_H),
                                             initial_state=s0.numpy(), d_final_state=dsn.numpy())
    for i, name in enumerate(("dq", "dk", "dv")):
        got = np.concatenate([np.load(os.path.join(tmp_path, f"cpb_{name}{r}.npy")) for r in range(world)], axis=1)
        np.testing.assert_allclose(got, want[i], rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(np.load(os.path.join(tmp_path, "cpb_ds00.npy")), want[3], rtol=1e-11, atol=1e-11)


def test_bench_launcher_starts_its_own_ranks():
    """bench.py --gpus N without a launcher starts N ranks itself: two gloo ranks of a stubbed step come up,
    and one JSON line reports the two ranks that ran (n_gpus, whole-job value over the slowest rank's time,
    and a config whose batch and parallelism are those of two ranks)."""
    import json

    import bench
    stub = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bench_rank_stub.py")
    status, out = bench.spawn_ranks(2, [], script=stub, capture=True, timeout_s=180)
    assert status == 0, out
    lines = [json.loads(x) for x in out.splitlines() if x.startswith("{")]
    assert len(lines) == 1, out
    d = lines[0]
    assert d["n_gpus"] == 2 and d["ms_per_step"] == 3.0
    assert d["value"] == 2 * 4 * 4096 / 3.0e-3
    assert d["config"]["global_batch"] == 8 and d["config"]["parallelism"] == "dp2"


def test_bench_gpus_flag_spawns_ranks_when_no_launcher(monkeypatch):
    """Without WORLD_SIZE in the environment, bench.main() hands --gpus N to the launcher and returns its
    status (nothing else runs in the parent process)."""
    import sys

    import bench
    calls = []
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench, "spawn_ranks", lambda n, argv, **kw: (calls.append((n, list(argv))) or (0, None)))
    monkeypatch.setattr(sys, "argv", ["bench.py", "--gpus", "4", "--steps", "3"])
    assert bench.main() == 0
    assert calls == [(4, ["--gpus", "4", "--steps", "3"])]


# --------------------------------------------------------------------------- context parallelism over varlen batches
# A packed batch cut into R equal shards along its token axis: sequences cross 0, 1 or several shard boundaries,
# some are empty (one at a boundary, one at the very end), and one boundary falls exactly between two sequences.
VCP_H, VCP_D = 2, 8
VCP_LENGTHS = (30, 0, 95, 7, 0, 44, 60, 3, 0)   # T = 239, padded below to 240 (a multiple of 1, 2, 3, 4, 8)


def _vcp_batch(R):
    lengths = list(VCP_LENGTHS)
    T = sum(lengths)
    pad = (-T) % 24
    lengths[-2] += pad               # T = 240; with R = 8 (L = 30): sequence 0 is exactly shard 0, the empty
                                     # sequence 1 sits on a boundary, sequence 2 crosses three boundaries and
                                     # sequence 6 two, and the empty last sequence sits at T
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    from linear_attention_hybrid_b200 import inputs as W
    T = int(cu[-1])
    q, k, v = (x.double() for x in W.make_qkv((T,), VCP_H, VCP_D, seed=21))
    g = W.make_grad_out((T,), VCP_H, VCP_D, seed=22).double()
    nseq = len(lengths)
    s0 = W.make_state((nseq,), VCP_H, VCP_D, VCP_D, std=0.1, seed=23).double()
    dsn = W.make_state((nseq,), VCP_H, VCP_D, VCP_D, std=0.1, seed=24).double()
    return cu, (q, k, v, g), s0, dsn


def test_varlen_shard_plan_partitions_every_sequence():
    """Brute force: over the ranks, the sub-sequences of every sequence tile exactly its tokens in order, every
    empty sequence is planned on exactly one rank, the local cu_seqlens cover each shard, and the continuation
    flags say whether a rank's first / last sub-sequence reaches past its shard."""
    from linear_attention_hybrid_b200.binding import VarlenShard
    rng = np.random.default_rng(3)
    for trial in range(200):
        nseq = int(rng.integers(1, 9))
        lengths = rng.integers(0, 40, size=nseq) * (rng.random(nseq) > 0.25)
        R = int(rng.choice([1, 2, 3, 4, 8]))
        T = int(lengths.sum())
        lengths[-1] += (-T) % R + (R if T + (-T) % R == 0 else 0)
        cu = np.concatenate([[0], np.cumsum(lengths)])
        T = int(cu[-1])
        L = T // R
        covered = {i: [] for i in range(nseq)}
        for r in range(R):
            sh = VarlenShard(cu, R, r)
            assert sh.local_cu[-1] == L and sh.local_cu[0] == 0
            assert all(b2 >= a2 for a2, b2 in zip(sh.local_cu, sh.local_cu[1:]))
            for (i, a, b), st, en in zip(sh.subs, sh.starts_here, sh.ends_here):
                assert r * L <= a <= b <= (r + 1) * L
                covered[i].append((a, b))
                assert st == (a == cu[i]) and en == (b == cu[i + 1])
            assert sh.first_continues == (cu[sh.seqs[0]] < r * L)
            assert sh.last_continues == (cu[sh.seqs[-1] + 1] > (r + 1) * L)
        for i in range(nseq):
            parts = covered[i]
            if cu[i] == cu[i + 1]:
                assert parts == [(cu[i], cu[i])]
            else:
                assert parts[0][0] == cu[i] and parts[-1][1] == cu[i + 1]
                assert all(p[1] == n[0] for p, n in zip(parts, parts[1:]))
                assert all(a < b for a, b in parts)


class _OracleVarlenOps:
    """The per-rank steps of the varlen context-parallel calls, in the oracle (fp64): states from a zero start,
    the entry states from the definition (the state at a point is the decayed state at the sequence start plus,
    for every earlier part, its state from a zero start decayed over the tokens after it), varlen prefill and
    backward."""
    lam = None

    @classmethod
    def _l(cls):
        import oracle
        return oracle.decay(VCP_H)[:, None, None]

    @staticmethod
    def shard_state(k, v, slopes):
        import oracle
        z = np.zeros(tuple(k.shape))
        return torch.from_numpy(oracle.prefill_recurrent(z, k.numpy(), v.numpy(), lam=oracle.decay(VCP_H),
                                                         return_final_state=True)[1])

    @staticmethod
    def shard_state_reverse(q, dout, slopes):
        import oracle
        z = np.zeros(tuple(q.shape))
        return torch.from_numpy(oracle.prefill_backward_recurrent(q.numpy(), z, z, dout.numpy(),
                                                                  lam=oracle.decay(VCP_H))[3])

    @classmethod
    def varlen_entry_state(cls, gathered, rank, cu, initial_state, slopes):
        cu = [int(x) for x in cu]
        R = gathered.shape[0]
        L = cu[-1] // R
        s = rank * L
        i = max(j for j in range(len(cu) - 1) if cu[j] <= s < cu[j + 1])
        if cu[i] == s:      # the first part starts its sequence: the first sequence at token s
            first = min(j for j in range(len(cu) - 1) if cu[j] == s)
            return torch.zeros(gathered.shape[1:], dtype=torch.float64) if initial_state is None else initial_state[first]
        out = np.zeros(tuple(gathered.shape[1:])) if initial_state is None else \
            cls._l() ** (s - cu[i]) * initial_state[i].numpy()
        for rp in range(R):
            a, b = max(cu[i], rp * L), min(cu[i + 1], (rp + 1) * L)
            if a < b and b <= s:
                out = out + cls._l() ** (s - b) * gathered[rp].numpy()
        return torch.from_numpy(out)

    @classmethod
    def varlen_reverse_entry_state(cls, gathered, rank, cu, d_final_state, slopes):
        cu = [int(x) for x in cu]
        R = gathered.shape[0]
        L = cu[-1] // R
        e = (rank + 1) * L
        i = max(j for j in range(len(cu) - 1) if cu[j] <= e - 1 < cu[j + 1])
        if cu[i + 1] == e:  # the last part ends its sequence (on the last rank the empty ones at T come after it)
            last = len(cu) - 2 if e == cu[-1] else i
            return torch.zeros(gathered.shape[1:], dtype=torch.float64) if d_final_state is None else d_final_state[last]
        out = np.zeros(tuple(gathered.shape[1:])) if d_final_state is None else \
            cls._l() ** (cu[i + 1] - e) * d_final_state[i].numpy()
        for rp in range(R):
            a, b = max(cu[i], rp * L), min(cu[i + 1], (rp + 1) * L)
            if a < b and a >= e:
                out = out + cls._l() ** (a - e) * gathered[rp].numpy()
        return torch.from_numpy(out)

    @staticmethod
    def prefill_varlen(q, k, v, local_cu, init, slopes, out_dtype):
        import oracle
        o, s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), cu_seqlens=local_cu, lam=oracle.decay(VCP_H),
                                        initial_state=init.numpy(), return_final_state=True)
        return torch.from_numpy(o), torch.from_numpy(s)

    @staticmethod
    def backward_varlen(q, k, v, dout, local_cu, init, dfin, slopes, out_dtype):
        import oracle
        return tuple(torch.from_numpy(x) for x in oracle.prefill_backward_recurrent(
            q.numpy(), k.numpy(), v.numpy(), dout.numpy(), cu_seqlens=local_cu, lam=oracle.decay(VCP_H),
            initial_state=init.numpy(), d_final_state=dfin.numpy()))


def _vcp_emulate(R):
    """Every rank's steps of la_prefill_varlen_cp and la_prefill_varlen_cp_backward in one process (the
    all-gather is a stack of the per-rank contributions), with the oracle doing the per-rank steps."""
    from linear_attention_hybrid_b200.binding import VarlenShard, varlen_cp_backward, varlen_cp_forward, varlen_cp_send
    cu, (q, k, v, g), s0, dsn = _vcp_batch(R)
    L = int(cu[-1]) // R
    shards = [VarlenShard(cu, R, r) for r in range(R)]
    loc = [tuple(x[r * L:(r + 1) * L].contiguous() for x in (q, k, v, g)) for r in range(R)]
    ops = _OracleVarlenOps
    fwd = torch.stack([varlen_cp_send(lk, lv, sh, ops=ops) for (lq, lk, lv, lg), sh in zip(loc, shards)])
    both = torch.stack([varlen_cp_send(lk, lv, sh, ops=ops, q=lq, dout=lg) for (lq, lk, lv, lg), sh in zip(loc, shards)])
    outs = [varlen_cp_forward(lq, lk, lv, sh, fwd, s0, True, ops=ops) for (lq, lk, lv, lg), sh in zip(loc, shards)]
    grads = [varlen_cp_backward(lq, lk, lv, lg, sh, both, s0, dsn, ops=ops)
             for (lq, lk, lv, lg), sh in zip(loc, shards)]
    return cu, (q, k, v, g), s0, dsn, outs, grads


@pytest.mark.parametrize("R", [1, 2, 3, 4, 8])
def test_varlen_context_parallel_emulated_ranks_equal_one_call(R):
    import oracle
    oracle.build()
    cu, (q, k, v, g), s0, dsn, outs, grads = _vcp_emulate(R)
    lam = oracle.decay(VCP_H)
    want_o, want_s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), cu_seqlens=cu, lam=lam,
                                              initial_state=s0.numpy(), return_final_state=True)
    np.testing.assert_allclose(torch.cat([o for o, _, _ in outs]).numpy(), want_o, rtol=1e-11, atol=1e-12)
    ended = {}
    for _, fin, ids in outs:
        for j, i in enumerate(ids):
            assert i not in ended
            ended[i] = fin[j].numpy()
    assert sorted(ended) == list(range(len(cu) - 1))   # every sequence ends on exactly one rank
    for i, s in ended.items():
        np.testing.assert_allclose(s, want_s[i], rtol=1e-11, atol=1e-12)
    want = oracle.prefill_backward_recurrent(q.numpy(), k.numpy(), v.numpy(), g.numpy(), cu_seqlens=cu, lam=lam,
                                             initial_state=s0.numpy(), d_final_state=dsn.numpy())
    for n, name in enumerate(("dq", "dk", "dv")):
        np.testing.assert_allclose(torch.cat([x[n] for x in grads]).numpy(), want[n], rtol=1e-10, atol=1e-12,
                                   err_msg=name)
    started = {}
    for *_, dinit, ids in grads:
        for j, i in enumerate(ids):
            assert i not in started
            started[i] = dinit[j].numpy()
    assert sorted(started) == list(range(len(cu) - 1))
    for i, d in started.items():
        np.testing.assert_allclose(d, want[3][i], rtol=1e-10, atol=1e-12)


def _vcp_rank_main(rank, world, port, out_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from linear_attention_hybrid_b200.binding import la_prefill_varlen_cp, la_prefill_varlen_cp_backward
        cu, (q, k, v, g), s0, dsn = _vcp_batch(world)
        L = int(cu[-1]) // world
        sl = slice(rank * L, (rank + 1) * L)
        o, fin, ids = la_prefill_varlen_cp(q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), cu,
                                           initial_state=s0, return_final_state=True, ops=_OracleVarlenOps)
        dq, dk, dv, dinit, sids = la_prefill_varlen_cp_backward(
            q[sl].contiguous(), k[sl].contiguous(), v[sl].contiguous(), g[sl].contiguous(), cu, initial_state=s0,
            d_final_state=dsn, ops=_OracleVarlenOps)
        np.savez(os.path.join(out_dir, f"vcp{rank}.npz"), o=o.numpy(), fin=fin.numpy(), ids=np.array(ids),
                 dq=dq.numpy(), dk=dk.numpy(), dv=dv.numpy(), dinit=dinit.numpy(), sids=np.array(sids))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_varlen_context_parallel_orchestration_on_two_ranks(tmp_path):
    """la_prefill_varlen_cp and la_prefill_varlen_cp_backward on two gloo ranks (the real all-gather), the oracle
    doing the per-rank steps: outputs, gradients, final states and initial-state gradients equal one call."""
    import oracle
    oracle.build()
    world = 2
    mp.start_processes(_vcp_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    cu, (q, k, v, g), s0, dsn = _vcp_batch(world)
    lam = oracle.decay(VCP_H)
    want_o, want_s = oracle.prefill_recurrent(q.numpy(), k.numpy(), v.numpy(), cu_seqlens=cu, lam=lam,
                                              initial_state=s0.numpy(), return_final_state=True)
    want = oracle.prefill_backward_recurrent(q.numpy(), k.numpy(), v.numpy(), g.numpy(), cu_seqlens=cu, lam=lam,
                                             initial_state=s0.numpy(), d_final_state=dsn.numpy())
    res = [np.load(os.path.join(tmp_path, f"vcp{r}.npz")) for r in range(world)]
    np.testing.assert_allclose(np.concatenate([x["o"] for x in res]), want_o, rtol=1e-11, atol=1e-12)
    for n, name in enumerate(("dq", "dk", "dv")):
        np.testing.assert_allclose(np.concatenate([x[name] for x in res]), want[n], rtol=1e-10, atol=1e-12)
    for x in res:
        for j, i in enumerate(x["ids"]):
            np.testing.assert_allclose(x["fin"][j], want_s[i], rtol=1e-11, atol=1e-12)
        for j, i in enumerate(x["sids"]):
            np.testing.assert_allclose(x["dinit"][j], want[3][i], rtol=1e-10, atol=1e-12)
