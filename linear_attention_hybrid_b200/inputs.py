"""Seeded synthetic inputs for the Lightning Attention workloads.

This module is the one place both the CUDA path's tests / benchmark and the
oracle are fed from. It holds none of the operator's arithmetic: it only draws
random numbers, scales them by 1/sqrt(D), optionally L2-normalises k per
(token, head), and rounds to the storage dtype.

Recipe (the pages print no workload for the operator; these are the specified
synthetic shapes, with the 256K context of the report's mid-training stage,
blog post news.neo-ai.one/en/article/3021, section "9.6T Tokens Continuous
Training", as the longest length):
  * q, k, v ~ iid N(0, 1) / sqrt(D), drawn in the order q, k, v from one
    ``torch.Generator`` seeded with ``seed``, as fp32, then cast to the dtype;
  * long-context workload: k L2-normalised over D per (token, head), in fp32,
    before the cast;
  * decode: state ~ iid N(0, 0.1^2) (std 0.1) in fp32 from seed ``seed``; the
    q, k, v of step ``i`` come from a generator seeded with
    ``decode_step_seed(seed, i)``, so any step can be regenerated alone;
  * varlen: lengths ``numpy.random.default_rng(seed).integers(lo, hi + 1, n)``;
  * backward pass: the output gradient dO ~ iid N(0, 1) / sqrt(D) from its own
    seed, and the final-state gradient like a state (std 0.1);
  * fused output norm + gate: gate pre-activation ~ iid N(0, 1), norm weight
    ~ 1 + 0.1 N(0, 1) per channel, eps = 1e-6.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_qkv(shape_lead, H: int, D: int, dtype=torch.bfloat16, seed: int = 0, device="cpu",
             k_l2norm: bool = False):
    """q, k, v with shape [*shape_lead, H, D], iid N(0,1)/sqrt(D) (k optionally L2-normalised)."""
    shape = tuple(shape_lead) + (H, D)
    g = _gen(seed, device)
    scale = 1.0 / math.sqrt(D)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * scale
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * scale
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32) * scale
    if k_l2norm:
        k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def make_grad_out(shape_lead, H: int, D: int, dtype=torch.bfloat16, seed: int = 0, device="cpu"):
    """The output gradient dO of a backward pass, [*shape_lead, H, D], iid N(0,1)/sqrt(D) (its own seed)."""
    g = _gen(seed, device)
    x = torch.randn(tuple(shape_lead) + (H, D), generator=g, device=device, dtype=torch.float32)
    return (x / math.sqrt(D)).to(dtype)


def make_norm_gate(shape_lead, H: int, D: int, dtype=torch.bfloat16, seed: int = 0, device="cpu"):
    """Inputs of the fused output norm + gate: the gate pre-activation z [*shape_lead, H, D] ~ iid N(0, 1) in
    `dtype`, and the norm weight [H, D] fp32 ~ 1 + 0.1 N(0, 1) (a trained scale near its unit init)."""
    g = _gen(seed, device)
    z = torch.randn(tuple(shape_lead) + (H, D), generator=g, device=device, dtype=torch.float32).to(dtype)
    w = 1.0 + 0.1 * torch.randn((H, D), generator=g, device=device, dtype=torch.float32)
    return z, w


def varlen_lengths(nseq: int = 8, lo: int = 1024, hi: int = 65536, seed: int = 0) -> np.ndarray:
    """Sequence lengths drawn uniformly from the integers lo..hi (both ends inclusive)."""
    return np.random.default_rng(seed).integers(lo, hi + 1, size=nseq).astype(np.int64)


def cu_seqlens_of(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def make_state(lead, H: int, Dk: int, Dv: int, std: float = 0.1, seed: int = 0, device="cpu"):
    """fp32 state [*lead, H, Dk, Dv] with iid N(0, std^2) entries."""
    g = _gen(seed, device)
    return torch.randn(tuple(lead) + (H, Dk, Dv), generator=g, device=device, dtype=torch.float32) * std


def decode_step_seed(seed: int, step: int) -> int:
    """Seed of the q, k, v drawn for decode step ``step`` (independent of every other step)."""
    return (int(seed) + 1) * 1_000_003 + int(step)


def make_decode_qkv(B: int, H: int, D: int, step: int, dtype=torch.bfloat16, seed: int = 0, device="cpu"):
    return make_qkv((B,), H, D, dtype=dtype, seed=decode_step_seed(seed, step), device=device)


@dataclass(frozen=True)
class Workload:
    """One of the five specified workloads (sizes only; inputs come from the functions above)."""
    name: str
    kind: str                     # "prefill" | "decode" | "varlen"
    H: int
    D: int
    dtype: torch.dtype
    B: int = 1
    N: int = 0
    steps: int = 0
    k_l2norm: bool = False
    lengths: tuple = field(default_factory=tuple)
    chain: tuple = field(default_factory=tuple)   # lengths of calls chained through the state
    return_final_state: bool = False
    seed: int = 0


def workloads():
    lens = tuple(int(x) for x in varlen_lengths(8, 1024, 65536, seed=0))
    return {
        "tiny_fp32": Workload("tiny_fp32", "prefill", H=2, D=64, dtype=torch.float32, B=1, N=256),
        "prefill_b4_n4096": Workload("prefill_b4_n4096", "prefill", H=16, D=128, dtype=torch.bfloat16,
                                     B=4, N=4096, return_final_state=True),
        "long_n65536": Workload("long_n65536", "prefill", H=16, D=128, dtype=torch.bfloat16, B=1, N=65536,
                                k_l2norm=True),
        "decode_b256": Workload("decode_b256", "decode", H=16, D=128, dtype=torch.bfloat16, B=256, steps=1000),
        "varlen_256k": Workload("varlen_256k", "varlen", H=16, D=128, dtype=torch.bfloat16, lengths=lens,
                                chain=(65536, 65536, 65536, 65536)),
    }
