#!/usr/bin/env python
"""Lightning Attention benchmark on B200: prefill tokens/s and TFLOP/s (H=16, D=128), decode state GB/s.

    python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl ours|reference]

One step is one call of the library's prefill over the workload's whole batch
(plan for packed batches, segment-state pass and chunk kernel: every kernel of
the prefill path; decode is timed in its own loop). Inputs are seeded synthetic
tensors resident in HBM before the timed region; they are larger than the
126 MB L2, so no flush is needed between steps. Timing uses CUDA events on the
launching stream, after W warm-up steps, bracketed by a barrier and a device
synchronize; for N > 1 every rank runs its own batch (weak scaling, no
collective on the data path) and the slowest rank's time is used.

Printed on rank 0 as one JSON line. Extra keys beyond the contract:
  tflops_alg / tflops_exec   algorithmic (causal triangle at C0 = 64) and executed (C = 128) FLOP rate
  step_hbm_frac              algorithmic bytes of the whole step / step time / measured HBM bandwidth
  kernels                    per-kernel mean milliseconds per step (library tracing, second pass)
  decode                     one decode step over 256 x 16 heads: us/step, GB/s and fraction of HBM
  workloads                  the other specified workloads, each timed the same way: long_n65536,
                             varlen_256k, the 4 x 65536 chained calls, and decode_b256 over its 1000 steps

--gpus N without a launcher starts N ranks itself (torch.distributed.run on 127.0.0.1); under a
launcher the ranks it started are used, and n_gpus, value and config always describe the ranks
that ran.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
KERNEL_SOURCES = ["linear_attention_hybrid_b200/csrc/la_chunk_tc.cuh", "linear_attention_hybrid_b200/csrc/la_ptx.cuh"]
TRAFFIC_FILE = "profiles/la_chunk_tc_kernel.traffic.json"
METRIC = "Lightning Attn prefill tokens/s & TFLOP/s (H16,D128); decode state GB/s"
# bf16 q, k, v in, fp16 o out: the configuration the full-size parity tests check against the bound
OUT_DTYPE = None  # set in main() (torch is imported lazily)
ALL_OUT = ()       # the output types the run times, set in main()


def pick_workload(W, args):
    """The workload timed: one of the specified ones, at another head dimension if --head-dim asks."""
    wl = W.workloads()[args.workload]
    if args.head_dim is not None and args.head_dim != wl.D:
        wl = dataclasses.replace(wl, D=args.head_dim, name=f"{wl.name}_d{args.head_dim}")
    return wl


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="prefill_b4_n4096",
                   choices=["prefill_b4_n4096", "long_n65536", "varlen_256k"])
    p.add_argument("--head-dim", type=int, choices=[64, 128], default=None,
                   help="run the workload's shape at this head dimension (named <workload>_d<D> when it differs)")
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-other-dtypes", action="store_true", help="skip the bf16- and fp32-output loops")
    p.add_argument("--no-backward", action="store_true", help="skip the backward-pass loop")
    p.add_argument("--no-norm-gate", action="store_true", help="skip the fused output norm + gate loops")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the other workloads' loops (long context, varlen, chained calls, 1000-step decode)")
    p.add_argument("--mode", choices=["dp", "cp"], default="dp",
                   help="dp: every rank its own batch (weak scaling, the default); cp: the long_n65536 sequence "
                        "sharded along N over the ranks (context parallelism, strong scaling)")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    return p.parse_args()


# --------------------------------------------------------------------------- peaks and clocks
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, read through NVML (read-only queries) every 5 ms
    by a helper thread while a timed loop runs: `with sampler.timing(): <timed loop>`. NVML is
    initialised before the first timed loop so that short loops still get samples; every timed loop
    of the run (prefill, end-to-end, decode, other output types) contributes."""
    REASONS = (("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("sw_power_cap", 0x4))
    PERIOD_S = 0.005

    def __init__(self, indices):
        import threading
        self.samples = []
        self.max_mhz = None
        self.error = None
        self.handles = []
        self.active = threading.Event()
        self.stop = threading.Event()
        try:
            import pynvml
            self.nvml = pynvml
            pynvml.nvmlInit()
            self.handles = [pynvml.nvmlDeviceGetHandleByIndex(i) for i in indices]
            self.max_mhz = max(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM) for h in self.handles)
        except Exception as e:  # NVML unavailable: report it rather than guess
            self.error = repr(e)
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _sample(self):
        nv = self.nvml
        for h in self.handles:
            mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            try:
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
            except Exception:
                bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
            self.samples.append((mhz, bits))

    def _run(self):
        try:
            while not self.stop.is_set():
                if self.active.wait(0.05):
                    self._sample()
                    self.stop.wait(self.PERIOD_S)
        except Exception as e:
            self.error = repr(e)

    def timing(self):
        import contextlib
        sampler = self

        @contextlib.contextmanager
        def region():
            sampler.active.set()
            try:
                yield
            finally:
                sampler.active.clear()
        return region()

    def close(self):
        self.stop.set()
        if self.handles:
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.error or "no samples"}
        reasons = sorted({name for _, bits in self.samples for name, bit in self.REASONS if bits & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "min_mhz": min(m for m, _ in self.samples), "reasons": reasons, "samples": len(self.samples),
                "source": "nvml every 5 ms during the timed loops"}


class _NoSampler:
    def timing(self):
        import contextlib
        return contextlib.nullcontext()

    def close(self):
        pass

    def summary(self):
        return None


# --------------------------------------------------------------------------- multi-rank helpers
# Weak scaling: every rank runs its own batch (independent sequences and heads, no exchange on the
# data path); the slowest rank's time is the job's time.
def rank_seed(seed, rank):
    """Seed of a rank's synthetic batch: distinct per rank, so the ranks process different data."""
    return seed + rank


def max_over_ranks(x, world, device):
    """The maximum of a per-rank scalar over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world, units_per_rank, ms):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank / (ms * 1e-3)


def free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(nprocs, argv, script=None, capture=False, timeout_s=None):
    """Run `script` (this file by default) with arguments `argv` as `nprocs` ranks of one node through
    torch.distributed.run, rendezvous on 127.0.0.1 at a free port. The ranks inherit this process's
    stdout, so rank 0's JSON line is the run's output (or, with capture=True, is returned in the output
    text). Returns (exit status, captured stdout or None)."""
    import subprocess
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", str(nprocs),
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), script or os.path.abspath(__file__),
           *argv]
    env = dict(os.environ)
    for key in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        env.pop(key, None)
    r = subprocess.run(cmd, env=env, stdout=subprocess.PIPE if capture else None, text=True, timeout=timeout_s)
    return r.returncode, (r.stdout if capture else None)


def init_ranks(backend="nccl", timeout_s=120):
    """(world, rank, local rank) from the launcher's environment; with more than one rank, the process group
    is initialised (NCCL: bound to this rank's GPU; gloo for CPU runs)."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        from datetime import timedelta
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def contract_line(value, world, steps, warmup, ms, config, **extra):
    """The JSON line's contract keys for a weak-scaling prefill run of `world` ranks (the whole job's
    tokens/s over the slowest rank's ms per step), followed by `extra`."""
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": steps,
            "warmup": warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1)/sqrt(D) inputs)",
            "config": config}
    line.update(extra)
    return line


def physical_indices(world):
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [int(x) for x in vis.split(",") if x.strip().isdigit()]
        return ids[:world] if ids else list(range(world))
    return list(range(world))


# --------------------------------------------------------------------------- workload arithmetic
def per_token_head_flops_alg(D):
    return 4 * D * D + 2 * 64 * D          # state update + inter (4D^2) and the causal triangle at C0 = 64


def per_token_head_flops_exec(D, C=128):
    return 4 * D * D + 4 * C * D           # four C x C x D / C x D x D tensor-core products per chunk


def traffic_for_current_kernel():
    """DRAM bytes per launch of the chunk kernel from the committed ncu summary, if the kernel is unchanged."""
    try:
        with open(os.path.join(ROOT, TRAFFIC_FILE)) as f:
            d = json.load(f)
        h = hashlib.sha256()
        for p in KERNEL_SOURCES:
            with open(os.path.join(ROOT, p), "rb") as g:
                h.update(g.read())
        if d.get("source_sha256") == h.hexdigest():
            return d
    except Exception:
        pass
    return None


# --------------------------------------------------------------------------- oracle timing (CPU)
def time_oracle(wl, seconds_target, seed=0):
    """Time the fp64 recurrent oracle on a bounded sample of the workload, sized to take about
    `seconds_target` seconds: a prefix of one sequence (all heads) or, once a whole sequence is quick,
    a batch of whole sequences. Returns (tokens/s, sample description, cores)."""
    import oracle
    from linear_attention_hybrid_b200 import inputs as W

    cores = oracle.default_threads()
    H, D = wl.H, wl.D
    lam = oracle.decay(H)
    seq_len = wl.N if wl.N else int(max(wl.lengths))

    def run(b, n):
        q, k, v = W.make_qkv((b, n), H, D, seed=seed)
        q, k, v = (x.double().numpy() for x in (q, k, v))
        t0 = time.perf_counter()
        oracle.prefill_recurrent(q, k, v, lam=lam, return_final_state=True)
        return time.perf_counter() - t0

    n0 = min(256, seq_len)
    t0 = max(run(1, n0), 1e-4)
    n = int(min(seq_len, max(n0, n0 * seconds_target / t0)))
    b = 1
    if n == seq_len:
        per_seq = t0 * seq_len / n0
        b = int(max(1, min(64, round(seconds_target / per_seq))))
    dt = run(b, n)
    desc = (f"{b} sequence(s) x {n} tokens x {H} heads (D={D}) of the workload's shape, fp64 recurrent form, "
            f"{cores} threads")
    return b * n / dt, desc, cores


def reference_arm(args):
    """The oracle, as it stands, on the host cores: same metric, unit and config as our arm."""
    import torch.distributed as dist
    from linear_attention_hybrid_b200 import inputs as W

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = pick_workload(W, args)
    per_step = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    vals = []
    desc, cores = "", 0
    for i in range(args.warmup + args.steps):
        v, desc, cores = time_oracle(wl, per_step, seed=i)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, int(os.environ.get("WORLD_SIZE", args.gpus))),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    del dist
    return 0


def config_of(wl, world):
    """The workload's config for a run of `world` ranks, each with its own batch of the workload's shape."""
    if wl.kind == "varlen":
        return {"workload": wl.name, "lengths": list(wl.lengths), "H": wl.H, "D": wl.D, "dtype": "bf16",
                "global_tokens": int(sum(wl.lengths)) * world, "l2": "inputs larger than L2 (no flush)",
                "parallelism": f"dp{world}"}
    return {"workload": wl.name, "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D, "dtype": "bf16",
            "global_batch": wl.B * world, "seq_len": wl.N, "final_state": wl.return_final_state,
            "k_l2norm": wl.k_l2norm, "l2": "inputs larger than L2 (no flush)", "parallelism": f"dp{world}"}


# --------------------------------------------------------------------------- our arm
def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # --gpus N without a launcher: start the N ranks here (one process per GPU, NCCL)
        status, _ = spawn_ranks(args.gpus, sys.argv[1:])
        return status

    import torch
    import torch.distributed as dist

    global OUT_DTYPE, ALL_OUT
    OUT_DTYPE = torch.float16
    ALL_OUT = (torch.float16, torch.bfloat16, torch.float32)
    world, rank, local = init_ranks("nccl")
    if world != args.gpus and rank == 0:
        print(f"bench.py: {world} ranks were launched with --gpus {args.gpus}; reporting the {world} that ran",
              file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from linear_attention_hybrid_b200.build import build, needs_build
    if needs_build():
        if rank == 0:
            build()
        if world > 1:
            dist.barrier()
    from linear_attention_hybrid_b200 import binding, inputs as W
    from linear_attention_hybrid_b200 import (la_decode_step, la_decode_steps, la_get_device_error, la_last_launch_count, la_prefill,
                                              la_prefill_backward, la_prefill_varlen, la_prefill_varlen_backward,
                                              la_decode_steps_norm_gate, la_prefill_norm_gate,
                                              la_prefill_varlen_norm_gate, la_trace_collect, la_trace_enable)

    hbm_gbs, bf16_tf, bf16_tf_sust, peak_kind = peaks()
    if args.mode == "cp":
        return cp_arm(args, world, rank, dev)
    wl = pick_workload(W, args)
    H, D = wl.H, wl.D
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_ranks(x):
        return max_over_ranks(x, world, dev)

    # ---------------- inputs resident in HBM
    if wl.kind == "varlen":
        lens = list(wl.lengths)
        cu = W.cu_seqlens_of(lens)
        T = int(cu[-1])
        q, k, v = W.make_qkv((T,), H, D, seed=rank_seed(wl.seed, rank), device=dev)
        cu_d = torch.tensor(cu, dtype=torch.int32, device=dev)
        nseq = len(lens)
        tokens = T
        o = torch.empty(q.shape, dtype=OUT_DTYPE, device=dev)
        sN = torch.empty((nseq, H, D, D), dtype=torch.float32, device=dev)
        # one workspace for every output type this run times (the work split depends on it)
        ws = torch.empty(max(1, max(binding.la_prefill_varlen_workspace_size(T, nseq, H, D, out_dtype=t) for t in ALL_OUT)),
                         dtype=torch.uint8, device=dev)

        def step(qq=q, kk=k, vv=v, oo=o, ss=sN):
            la_prefill_varlen(qq, kk, vv, cu_d, final_state=ss, o=oo, workspace=ws)
        state_bytes = nseq * H * D * D * 4
    else:
        q, k, v = W.make_qkv((wl.B, wl.N), H, D, seed=rank_seed(wl.seed, rank), device=dev, k_l2norm=wl.k_l2norm)
        tokens = wl.B * wl.N
        o = torch.empty(q.shape, dtype=OUT_DTYPE, device=dev)
        sN = torch.empty((wl.B, H, D, D), dtype=torch.float32, device=dev)
        # one workspace for every output type this run times (the work split depends on it)
        ws = torch.empty(max(1, max(binding.la_prefill_workspace_size(wl.B, wl.N, H, D, out_dtype=t) for t in ALL_OUT)),
                         dtype=torch.uint8, device=dev)

        def step(qq=q, kk=k, vv=v, oo=o, ss=sN):
            la_prefill(qq, kk, vv, final_state=ss, o=oo, workspace=ws)
        state_bytes = wl.B * H * D * D * 4

    token_heads = tokens * H
    # q, k, v read as bf16, o written in OUT_DTYPE, final state written
    alg_bytes = token_heads * D * (3 * 2 + o.element_size()) + state_bytes
    flops_alg = token_heads * per_token_head_flops_alg(D)
    flops_exec = token_heads * per_token_head_flops_exec(D)

    sampler = ClockSampler(physical_indices(world)) if rank == 0 else _NoSampler()
    for _ in range(args.warmup):
        step()
    launches_per_step = la_last_launch_count()
    torch.cuda.synchronize()
    assert la_get_device_error() == 0

    # ---------------- timed region (device-resident inputs)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with sampler.timing():
        ev0.record(stream)
        h0 = time.perf_counter()
        for _ in range(args.steps):
            step()
        h1 = time.perf_counter()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = max_ranks(ev0.elapsed_time(ev1) / args.steps)
    host_us = (h1 - h0) / args.steps * 1e6   # the calls' own CPU time (they are asynchronous)

    value = weak_scaling_value(world, tokens, ms)
    tflops_alg = world * flops_alg / (ms * 1e-3) / 1e12
    tflops_exec = world * flops_exec / (ms * 1e-3) / 1e12

    # ---------------- per-kernel durations (second pass, library tracing on the same stream)
    la_trace_enable(True)
    for _ in range(args.steps):
        step()
    recs = la_trace_collect()
    la_trace_enable(False)
    per_kernel = {}
    for name, t in recs:
        per_kernel.setdefault(name, []).append(t)
    kernels = {n: {"ms_mean": statistics.mean(ts), "launches_per_step": len(ts) / args.steps}
               for n, ts in per_kernel.items()}
    dominant = max(per_kernel, key=lambda n: sum(per_kernel[n]))
    dom_ms = statistics.mean(per_kernel[dominant])
    achieved = alg_bytes / (dom_ms * 1e-3) / 1e9
    tr = traffic_for_current_kernel() if dominant == "la_chunk_tc_kernel" else None
    traffic = None
    if tr and tr.get("workload") == wl.name:
        traffic = tr.get("dram_bytes_per_launch")
    roofline = {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                "frac": achieved / hbm_gbs, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_kind == "measured" else "fallback", "traffic": traffic,
                "alg_bytes_per_launch": alg_bytes, "kernel_ms": dom_ms}

    # ---------------- end to end through the public API with host buffers: every step copies its inputs in
    #                  from pinned host memory and its output and final state back, as a serving loop would
    #                  run it: copy-in, compute and copy-back on three streams with two device buffer sets, so
    #                  that step i's copy-in overlaps step i-1's compute and copy-back (PCIe is full duplex)
    e2e = None
    if not args.no_e2e:
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        ho = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        hs = torch.empty(sN.shape, dtype=sN.dtype).pin_memory()
        bufs = [tuple(torch.empty_like(x) for x in (q, k, v, o, sN)) for _ in range(2)]
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        for b in range(2):   # every event recorded once, so that the first waits are satisfied
            for ev in (ev_in[b], ev_comp[b], ev_out[b]):
                ev.record(stream)

        def e2e_step(i):
            b = i % 2
            bq, bk, bv, bo, bs = bufs[b]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b])      # the compute that read this buffer set is done
                bq.copy_(hq, non_blocking=True)
                bk.copy_(hk, non_blocking=True)
                bv.copy_(hv, non_blocking=True)
                ev_in[b].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[b])
                s_comp.wait_event(ev_out[b])     # the copy-back that read this output is done
                step(bq, bk, bv, bo, bs)
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                ho.copy_(bo, non_blocking=True)
                hs.copy_(bs, non_blocking=True)
                ev_out[b].record(s_out)

        for i in range(max(2, min(4, args.warmup))):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        e2e_steps = max(8, args.steps)     # enough steps that the pipeline fill and drain are amortised
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with sampler.timing():
            e0.record(s_in)
            for i in range(e2e_steps):
                e2e_step(i)
            e1.record(s_out)
            torch.cuda.synchronize()
        barrier()
        ems = max_ranks(e0.elapsed_time(e1) / e2e_steps)
        h2d = 3 * q.numel() * q.element_size()
        d2h = o.numel() * o.element_size() + sN.numel() * sN.element_size()
        e2e = {"value": world * tokens / (ems * 1e-3), "unit": "tokens/s", "ms_per_step": ems,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "pipelining": "copy-in, compute and copy-back on three streams, two device buffer sets",
               "h2d_GB/s": h2d / (ems * 1e-3) / 1e9}
        del hq, hk, hv, ho, hs, bufs

    # ---------------- decode: one step over 256 sequences x 16 heads, state in place
    decode = None
    if not args.no_decode:
        dw = W.workloads()["decode_b256"]
        Sd = W.make_state((dw.B,), dw.H, dw.D, dw.D, std=0.1, seed=rank_seed(dw.seed, rank), device=dev)
        dq1, dk1, dv1 = W.make_decode_qkv(dw.B, dw.H, dw.D, step=0, seed=rank_seed(dw.seed, rank), device=dev)
        od = torch.empty(dq1.shape, dtype=OUT_DTYPE, device=dev)
        for _ in range(args.warmup):
            la_decode_step(dq1, dk1, dv1, Sd, o=od)
        torch.cuda.synchronize()
        barrier()
        dsteps = max(args.steps, 50)
        with sampler.timing():
            ev0.record(stream)
            for _ in range(dsteps):
                la_decode_step(dq1, dk1, dv1, Sd, o=od)
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier()
        dms = max_ranks(ev0.elapsed_time(ev1) / dsteps)
        dbytes = 2 * Sd.numel() * 4 + 3 * dq1.numel() * 2 + od.numel() * od.element_size()
        gbs = world * dbytes / (dms * 1e-3) / 1e9
        decode = {"workload": dw.name, "us_per_step": dms * 1e3, "GB/s": gbs, "frac_of_hbm": gbs / (world * hbm_gbs),
                  "bytes_per_step": dbytes, "steps_timed": dsteps}
        # several tokens per launch: the state is read and written once for all of them
        Kt = 8
        mq, mk, mv = W.make_qkv((dw.B, Kt), dw.H, dw.D, seed=rank_seed(dw.seed, rank), device=dev)
        mo = torch.empty(mq.shape, dtype=OUT_DTYPE, device=dev)
        for _ in range(args.warmup):
            la_decode_steps(mq, mk, mv, Sd, o=mo)
        torch.cuda.synchronize()
        barrier()
        mlaunches = max(args.steps, 20)
        with sampler.timing():
            ev0.record(stream)
            for _ in range(mlaunches):
                la_decode_steps(mq, mk, mv, Sd, o=mo)
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier()
        mms = max_ranks(ev0.elapsed_time(ev1) / mlaunches)
        mbytes = 2 * Sd.numel() * 4 + 3 * mq.numel() * 2 + mo.numel() * mo.element_size()
        decode["multi_token"] = {"tokens_per_launch": Kt, "us_per_launch": mms * 1e3,
                                 "tokens_per_s": world * dw.B * Kt / (mms * 1e-3),
                                 "GB/s": world * mbytes / (mms * 1e-3) / 1e9,
                                 "speedup_vs_single_steps": Kt * dms / mms}
        del Sd, mq, mk, mv, mo

    # ---------------- the same step with the other output types (bf16: rounded to 8 bits; fp32: unrounded)
    other_out = {}
    for name, odt in () if args.no_other_dtypes else (("bf16", torch.bfloat16), ("fp32", torch.float32)):
        ox = torch.empty(q.shape, dtype=odt, device=dev)
        for _ in range(args.warmup):
            step(q, k, v, ox, sN)
        torch.cuda.synchronize()
        barrier()
        with sampler.timing():
            ev0.record(stream)
            for _ in range(args.steps):
                step(q, k, v, ox, sN)
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier()
        msx = max_ranks(ev0.elapsed_time(ev1) / args.steps)
        bx = token_heads * D * (3 * 2 + ox.element_size()) + state_bytes
        other_out[name] = {"value": world * tokens / (msx * 1e-3), "unit": "tokens/s", "ms_per_step": msx,
                           "step_GB/s": bx / (msx * 1e-3) / 1e9, "step_hbm_frac": bx / (msx * 1e-3) / 1e9 / hbm_gbs}
        del ox

    # ---------------- backward pass of the same workload (training: zero initial state, no final-state
    #                  gradient; bf16 dq, dk, dv from bf16 q, k, v, dO)
    backward = None
    if not args.no_backward:
        g = W.make_grad_out(q.shape[:-2], H, D, seed=rank_seed(wl.seed, rank) + 1000, device=dev)
        gq, gk, gv = (torch.empty_like(x) for x in (q, k, v))
        if wl.kind == "varlen":
            bws = torch.empty(binding.la_prefill_varlen_backward_workspace_size(tokens, nseq, H, D), dtype=torch.uint8,
                              device=dev)

            def bstep():
                la_prefill_varlen_backward(q, k, v, g, cu_d, dq=gq, dk=gk, dv=gv, workspace=bws)
        else:
            bws = torch.empty(binding.la_prefill_backward_workspace_size(wl.B, wl.N, H, D), dtype=torch.uint8,
                              device=dev)

            def bstep():
                la_prefill_backward(q, k, v, g, dq=gq, dk=gk, dv=gv, workspace=bws)
        for _ in range(args.warmup):
            bstep()
        blaunches = la_last_launch_count()
        torch.cuda.synchronize()
        barrier()
        with sampler.timing():
            ev0.record(stream)
            for _ in range(args.steps):
                bstep()
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier()
        bms = max_ranks(ev0.elapsed_time(ev1) / args.steps)
        la_trace_enable(True)
        for _ in range(args.steps):
            bstep()
        brecs = la_trace_collect()
        la_trace_enable(False)
        bk = {}
        for name, t in brecs:
            bk.setdefault(name, []).append(t)
        # q, k, v, dO read and dq, dk, dv written once each: the floor of any implementation
        bbytes = token_heads * D * 2 * 7
        backward = {"workload": wl.name, "ms_per_step": bms, "tokens_per_s": world * tokens / (bms * 1e-3),
                    "alg_bytes_per_step": bbytes, "alg_GB/s": bbytes / (bms * 1e-3) / 1e9,
                    "frac_of_hbm": bbytes / (bms * 1e-3) / 1e9 / hbm_gbs, "launches_per_step": blaunches,
                    "kernels": {n: {"ms_total_per_step": sum(ts) / args.steps, "launches_per_step": len(ts) / args.steps}
                                for n, ts in bk.items()},
                    "vs_forward_step": bms / ms, "dtype": "bf16 in, bf16 gradients"}
        del g, gq, gk, gv, bws

    # ---------------- the fused output norm + gate (inference): the same prefill step and one decode step
    norm_gate = None
    if not args.no_norm_gate:
        z, wn = W.make_norm_gate(q.shape[:-2], H, D, seed=rank_seed(wl.seed, rank) + 2000, device=dev)
        if wl.kind == "varlen":
            def gstep():
                la_prefill_varlen_norm_gate(q, k, v, z, wn, cu_d, final_state=sN, o=o, workspace=ws)
        else:
            def gstep():
                la_prefill_norm_gate(q, k, v, z, wn, final_state=sN, o=o, workspace=ws)
        for _ in range(args.warmup):
            gstep()
        torch.cuda.synchronize()
        barrier()
        with sampler.timing():
            ev0.record(stream)
            for _ in range(args.steps):
                gstep()
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier()
        gms = max_ranks(ev0.elapsed_time(ev1) / args.steps)
        la_trace_enable(True)
        for _ in range(args.steps):
            gstep()
        grecs = [t for n, t in la_trace_collect() if n == "la_norm_gate_kernel"]
        la_trace_enable(False)
        nms = statistics.mean(grecs)
        nbytes = token_heads * D * (2 * o.element_size() + 2)   # o read, gate read, y written
        norm_gate = {"prefill": {"ms_per_step": gms, "tokens_per_s": world * tokens / (gms * 1e-3),
                                 "vs_plain_step": gms / ms},
                     "norm_gate_kernel": {"ms": nms, "alg_bytes": nbytes, "GB/s": nbytes / (nms * 1e-3) / 1e9,
                                          "frac_of_hbm": nbytes / (nms * 1e-3) / 1e9 / hbm_gbs}}
        del z, wn
        if decode is not None:
            dw = W.workloads()["decode_b256"]
            Sd = W.make_state((dw.B,), dw.H, dw.D, dw.D, std=0.1, seed=rank_seed(dw.seed, rank), device=dev)
            gq, gk, gv = W.make_qkv((dw.B, 1), dw.H, dw.D, seed=rank_seed(dw.seed, rank) + 1, device=dev)
            gz, gw = W.make_norm_gate((dw.B, 1), dw.H, dw.D, seed=rank_seed(dw.seed, rank) + 2, device=dev)
            go = torch.empty(gq.shape, dtype=OUT_DTYPE, device=dev)
            for _ in range(args.warmup):
                la_decode_steps_norm_gate(gq, gk, gv, gz, gw, Sd, o=go)
            torch.cuda.synchronize()
            barrier()
            dsteps = max(args.steps, 50)
            with sampler.timing():
                ev0.record(stream)
                for _ in range(dsteps):
                    la_decode_steps_norm_gate(gq, gk, gv, gz, gw, Sd, o=go)
                ev1.record(stream)
                torch.cuda.synchronize()
            barrier()
            gdms = max_ranks(ev0.elapsed_time(ev1) / dsteps)
            norm_gate["decode"] = {"us_per_step": gdms * 1e3, "vs_plain_step": gdms * 1e3 / decode["us_per_step"]}
            del Sd, gq, gk, gv, gz, gw, go

    # ---------------- the other specified workloads, each timed the same way (every rank its own batch):
    #                  the long-context prefill, the packed varlen batch, the 262144-token sequence as four
    #                  chained calls carrying the state, and the decode workload over all of its 1000 steps
    others = None
    if not args.no_workloads:
        others = {}

        def timed(fn, n):
            """Device ms per call (CUDA events), and host us per call: the time the loop of library calls
            itself takes on the CPU (the calls are asynchronous, so a host time at or above the device time
            means the loop, not the GPU, sets the step)."""
            for _ in range(max(1, args.warmup)):
                fn()
            torch.cuda.synchronize()
            barrier()
            with sampler.timing():
                ev0.record(stream)
                h0 = time.perf_counter()
                for _ in range(n):
                    fn()
                h1 = time.perf_counter()
                ev1.record(stream)
                torch.cuda.synchronize()
            barrier()
            return max_ranks(ev0.elapsed_time(ev1) / n), (h1 - h0) / n * 1e6

        def traced(fn, n):
            la_trace_enable(True)
            for _ in range(n):
                fn()
            recs = la_trace_collect()
            la_trace_enable(False)
            per = {}
            for name, t in recs:
                per.setdefault(name, []).append(t)
            return {nm: sum(ts) / n for nm, ts in per.items()}

        def entry(name, fn, tokens_x, bytes_x, n):
            msx, hostx = timed(fn, n)
            kx = traced(fn, n)
            dom = max(kx, key=kx.get)
            return {"workload": name, "ms_per_step": msx, "host_us_per_call": hostx,
                    "tokens_per_s": world * tokens_x / (msx * 1e-3),
                    "alg_bytes_per_step": bytes_x, "step_GB/s": bytes_x / (msx * 1e-3) / 1e9,
                    "step_hbm_frac": bytes_x / (msx * 1e-3) / 1e9 / hbm_gbs,
                    "kernels_ms_per_step": kx,
                    "roofline": {"kernel": dom, "frac": bytes_x / (kx[dom] * 1e-3) / 1e9 / hbm_gbs,
                                 "note": "algorithmic bytes of the whole step over the dominant kernel's time"}}

        n_other = max(5, min(args.steps, 10))
        for name in ("long_n65536", "varlen_256k"):
            if name == wl.name:
                continue
            xw = W.workloads()[name]
            if xw.kind == "varlen":
                xl = list(xw.lengths)
                xcu = torch.tensor(W.cu_seqlens_of(xl), dtype=torch.int32, device=dev)
                xT = int(sum(xl))
                xq, xk, xv = W.make_qkv((xT,), H, D, seed=rank_seed(xw.seed, rank), device=dev)
                xo = torch.empty(xq.shape, dtype=OUT_DTYPE, device=dev)
                xs = torch.empty((len(xl), H, D, D), dtype=torch.float32, device=dev)
                xws = torch.empty(max(1, binding.la_prefill_varlen_workspace_size(xT, len(xl), H, D, out_dtype=OUT_DTYPE)),
                                  dtype=torch.uint8, device=dev)

                def xfn(xq=xq, xk=xk, xv=xv, xo=xo, xs=xs, xws=xws, xcu=xcu):
                    la_prefill_varlen(xq, xk, xv, xcu, final_state=xs, o=xo, workspace=xws)
                xtok, xstates = xT, len(xl)
            else:
                xq, xk, xv = W.make_qkv((xw.B, xw.N), H, D, seed=rank_seed(xw.seed, rank), device=dev,
                                        k_l2norm=xw.k_l2norm)
                xo = torch.empty(xq.shape, dtype=OUT_DTYPE, device=dev)
                xs = torch.empty((xw.B, H, D, D), dtype=torch.float32, device=dev)
                xws = torch.empty(max(1, binding.la_prefill_workspace_size(xw.B, xw.N, H, D, out_dtype=OUT_DTYPE)), dtype=torch.uint8,
                                  device=dev)

                def xfn(xq=xq, xk=xk, xv=xv, xo=xo, xs=xs, xws=xws):
                    la_prefill(xq, xk, xv, final_state=xs, o=xo, workspace=xws)
                xtok, xstates = xw.B * xw.N, xw.B
            xbytes = xtok * H * D * (3 * 2 + 2) + xstates * H * D * D * 4
            others[name] = entry(name, xfn, xtok, xbytes, n_other)
            del xq, xk, xv, xo, xs, xws

        # the prefill workload's shape at the other head dimension, D = 64 (its own kernel instances), with
        # the final states returned
        pw = W.workloads()["prefill_b4_n4096"]
        D64 = 64
        xq, xk, xv = W.make_qkv((pw.B, pw.N), pw.H, D64, seed=rank_seed(pw.seed + 3, rank), device=dev)
        xo = torch.empty(xq.shape, dtype=OUT_DTYPE, device=dev)
        xs = torch.empty((pw.B, pw.H, D64, D64), dtype=torch.float32, device=dev)
        xws = torch.empty(max(1, binding.la_prefill_workspace_size(pw.B, pw.N, pw.H, D64, out_dtype=OUT_DTYPE)),
                          dtype=torch.uint8, device=dev)

        def d64fn(xq=xq, xk=xk, xv=xv, xo=xo, xs=xs, xws=xws):
            la_prefill(xq, xk, xv, final_state=xs, o=xo, workspace=xws)
        d64bytes = pw.B * pw.N * pw.H * D64 * (3 * 2 + 2) + pw.B * pw.H * D64 * D64 * 4
        others["prefill_b4_n4096_d64"] = entry("prefill_b4_n4096_d64", d64fn, pw.B * pw.N, d64bytes, n_other)
        del xq, xk, xv, xo, xs, xws

        # the 262144-token sequence of the varlen workload, run as four chained 65536-token calls: each call's
        # final state is the next call's initial state (one sequence, B = 1)
        vw = W.workloads()["varlen_256k"]
        Nc = sum(vw.chain)
        cq_, ck_, cv_ = W.make_qkv((1, Nc), H, D, seed=rank_seed(vw.seed + 1, rank), device=dev)
        parts, t0_ = [], 0
        for L in vw.chain:
            parts.append(tuple(x[:, t0_:t0_ + L].contiguous() for x in (cq_, ck_, cv_)))
            t0_ += L
        del cq_, ck_, cv_
        couts = [torch.empty(p_[0].shape, dtype=OUT_DTYPE, device=dev) for p_ in parts]
        cstate = [torch.zeros((1, H, D, D), dtype=torch.float32, device=dev) for _ in range(2)]
        cws = torch.empty(max(1, binding.la_prefill_workspace_size(1, vw.chain[0], H, D, out_dtype=OUT_DTYPE)), dtype=torch.uint8,
                          device=dev)

        def chain():
            for j, (pq, pk, pv) in enumerate(parts):
                la_prefill(pq, pk, pv, initial_state=None if j == 0 else cstate[(j + 1) % 2],
                           final_state=cstate[j % 2], o=couts[j], workspace=cws)
        cbytes = Nc * H * D * (3 * 2 + 2) + len(vw.chain) * H * D * D * 4 * 2
        others["chain_4x65536"] = entry("chain_4x65536", chain, Nc, cbytes, n_other)
        del parts, couts, cstate, cws

        # decode: all 1000 steps of the workload with the inputs of every step drawn in advance (resident in HBM)
        dw = W.workloads()["decode_b256"]
        Sd = W.make_state((dw.B,), dw.H, dw.D, dw.D, std=0.1, seed=rank_seed(dw.seed, rank), device=dev)
        dins = [W.make_decode_qkv(dw.B, dw.H, dw.D, step=i, seed=rank_seed(dw.seed, rank), device=dev)
                for i in range(dw.steps)]
        od = torch.empty(dins[0][0].shape, dtype=OUT_DTYPE, device=dev)

        def decode_all():
            for dq_, dk_, dv_ in dins:
                la_decode_step(dq_, dk_, dv_, Sd, o=od)
        for i in range(2):
            la_decode_step(*dins[i], Sd, o=od)
        torch.cuda.synchronize()
        barrier()
        with sampler.timing():
            ev0.record(stream)
            decode_all()
            ev1.record(stream)
            torch.cuda.synchronize()
        barrier()
        d_ms = max_ranks(ev0.elapsed_time(ev1))
        d_bytes = 2 * Sd.numel() * 4 + 3 * dins[0][0].numel() * 2 + od.numel() * od.element_size()
        others["decode_b256_1000_steps"] = {
            "workload": dw.name, "steps": dw.steps, "ms_total": d_ms, "us_per_step": d_ms * 1e3 / dw.steps,
            "bytes_per_step": d_bytes, "GB/s": world * d_bytes * dw.steps / (d_ms * 1e-3) / 1e9,
            "frac_of_hbm": d_bytes * dw.steps / (d_ms * 1e-3) / 1e9 / hbm_gbs,
            "inputs": "fresh q, k, v for every step (drawn in advance), state updated in place"}
        del Sd, dins, od

    assert la_get_device_error() == 0, "device status recorded during the benchmark"
    sampler.close()
    clocks = sampler.summary()

    # ---------------- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        val, desc, cores = time_oracle(wl, args.cpu_seconds)
        cpu = {"value": val, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = contract_line(
            value, world, args.steps, args.warmup, ms, config_of(wl, world),
            tflops_alg=tflops_alg, tflops_exec=tflops_exec,
            step_hbm_frac=alg_bytes / (ms * 1e-3) / 1e9 / hbm_gbs,
            roofline=roofline, cpu_baseline=cpu, e2e=e2e,
            gpu_launches=launches_per_step * args.steps, host_us_per_call=host_us,
            clocks=clocks, kernels=kernels, decode=decode, other_output_dtypes=other_out,
            backward=backward, norm_gate=norm_gate, workloads=others,
            output_dtype="fp16 o (bf16 q/k/v; fp32 accumulation and state)",
            tensor_frac_exec_of_burst_peak=tflops_exec / world / bf16_tf)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def cp_arm(args, world, rank, dev):
    """Context parallelism: the long_n65536 sequence (B=1, H=16) cut into `world` shards along N, rank r
    holding tokens [r*L, (r+1)*L); one step is la_prefill_cp on every rank (shard state pass, all-gather of
    the shard states, entry state, prefill). Strong scaling: the job's tokens are fixed."""
    import torch
    import torch.distributed as dist
    from linear_attention_hybrid_b200 import inputs as W
    from linear_attention_hybrid_b200 import la_get_device_error, la_last_launch_count, la_prefill_cp, la_prefill_cp_backward

    wl = W.workloads()["long_n65536"]
    N, H, D = wl.N, wl.H, wl.D
    if N % world:
        raise SystemExit(f"N={N} must be divisible by the {world} ranks")
    L = N // world
    q, k, v = W.make_qkv((wl.B, N), H, D, seed=wl.seed, device=dev, k_l2norm=wl.k_l2norm)  # one sequence
    sl = slice(rank * L, (rank + 1) * L)
    qs, ks, vs = (x[:, sl].contiguous() for x in (q, k, v))
    del q, k, v
    stream = torch.cuda.current_stream()
    launches = [0]

    def step():
        la_prefill_cp(qs, ks, vs, return_final_state=True, out_dtype=torch.float16)
        launches[0] = la_last_launch_count()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert la_get_device_error() == 0
    sampler = ClockSampler(physical_indices(world)) if rank == 0 else _NoSampler()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler.timing():
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world, dev)

    # the context-parallel backward pass of the same shards (training: zero initial state, no final-state
    # gradient): shard states forward and reversed, one all-gather, both entry states, the local backward
    g = W.make_grad_out((wl.B, N), H, D, seed=wl.seed + 1000, device=dev)[:, sl].contiguous()

    def bstep():
        la_prefill_cp_backward(qs, ks, vs, g)

    for _ in range(max(3, args.warmup)):
        bstep()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler.timing():
        ev0.record(stream)
        for _ in range(args.steps):
            bstep()
        ev1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    bms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world, dev)
    sampler.close()
    assert la_get_device_error() == 0
    if rank == 0:
        line = {
            "metric": METRIC, "value": wl.B * N / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1)/sqrt(D) inputs)",
            "config": {"workload": wl.name, "B": wl.B, "N": N, "H": H, "D": D, "dtype": "bf16",
                       "tokens_per_rank": L, "parallelism": f"cp{world}", "l2": "inputs larger than L2 (no flush)"},
            "mode": "context parallel (shard state pass, all-gather of shard states, entry state, prefill)",
            "backward": {"ms_per_step": bms, "tokens_per_s": wl.B * N / (bms * 1e-3),
                         "mode": "forward and reversed shard states, one all-gather, entry states, local backward"},
            "gpu_launches": None, "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
