"""One rank of bench.py's multi-rank path with a stubbed step, for the CPU launcher test.

bench.spawn_ranks starts this script as the ranks of one node (gloo on CPU): each rank
initialises the group with bench.init_ranks, "takes" 2 + rank milliseconds per step,
and the line is assembled exactly as bench.py's own arm assembles it (slowest rank's
time, whole-job throughput, the config of the ranks that ran), printed by rank 0 only.
"""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402
from linear_attention_hybrid_b200 import inputs as W  # noqa: E402


def main():
    world, rank, _ = bench.init_ranks("gloo", timeout_s=60)
    wl = W.workloads()["prefill_b4_n4096"]
    ms = bench.max_over_ranks(2.0 + rank, world, torch.device("cpu"))
    value = bench.weak_scaling_value(world, wl.B * wl.N, ms)
    if rank == 0:
        print(json.dumps(bench.contract_line(value, world, 3, 1, ms, bench.config_of(wl, world))), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
