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


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    """Under torchrun only rank 0 times the oracle and prints; the other ranks exit 0 at once."""
    import argparse

    import bench
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(workload="prefill_b4_n4096", steps=1, warmup=0, gpus=2)
    assert bench.reference_arm(args) == 0
