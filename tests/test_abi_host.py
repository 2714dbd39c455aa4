"""Host-side checks of the C ABI that need no GPU: the library builds for
sm_100a, loads, exports every function include/la.h declares, and rejects bad
arguments before touching CUDA (fake, never-dereferenced device pointers)."""

import ctypes
import os
import re

import pytest
import torch

from linear_attention_hybrid_b200 import binding
from linear_attention_hybrid_b200.build import INCLUDE, build

LA_BF16, LA_FP32, LA_BF16_F32OUT, LA_BF16_F16OUT = 0, 1, 2, 3


@pytest.fixture(scope="module")
def L():
    build()
    return binding.lib()


def _declared_functions():
    with open(os.path.join(INCLUDE, "la.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(la_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    declared = _declared_functions()
    assert declared, "no declarations found"
    assert set(declared) == set(binding.EXPORTS)
    for name in declared:
        assert hasattr(L, name), f"{name} not exported"


def test_library_has_no_cuda_runtime_dependency():
    # the runtime is linked statically: the library loads on a machine without the toolkit's shared libs
    out = os.popen(f"ldd {binding.LIB_PATH}").read()
    assert "libcudart" not in out and "libcuda.so" not in out


def test_status_strings(L):
    for code, name in enumerate(["LA_OK", "LA_ERR_INVALID_ARGUMENT", "LA_ERR_UNSUPPORTED", "LA_ERR_WORKSPACE",
                                 "LA_ERR_CUDA", "LA_ERR_DEVICE_TIMEOUT"]):
        assert L.la_status_string(code).decode() == name


def test_workspace_sizes(L):
    # the tensor-core path plans a segment split for small batches: plan arrays + one fp32 state per unit/head
    ws = L.la_prefill_workspace_size(4, 4096, 16, 128, LA_BF16)
    assert ws >= 4 * 16 * 128 * 128 * 4
    assert L.la_prefill_workspace_size(4, 4096, 16, 128, LA_FP32) == 0      # CUDA-core path needs none
    # D = 64 with bf16 inputs runs in the tensor-core kernels' 128-wide tiles: the same plan as D = 128, with
    # the segment states in 128 x 128 tiles and only the initial-state copies in the caller's 64 x 64
    w64, w128 = L.la_prefill_workspace_size(1, 4096, 2, 64, LA_BF16), L.la_prefill_workspace_size(1, 4096, 2, 128, LA_BF16)
    assert w64 > 0 and w128 - w64 == 1 * 2 * (128 * 128 - 64 * 64) * 4
    # fp16 / fp32 outputs take the corrected split: the segments' exit states in 128 x 128 tiles whatever D,
    # no copy of the initial state
    c64 = L.la_prefill_workspace_size(1, 4096, 2, 64, LA_BF16_F16OUT)
    c128 = L.la_prefill_workspace_size(1, 4096, 2, 128, LA_BF16_F32OUT)
    assert c64 > 0 and c64 == c128 and c128 % (2 * 128 * 128 * 4) == 0
    assert L.la_prefill_workspace_size(1, 256, 2, 64, LA_FP32) == 0        # fp32 runs on the CUDA cores
    assert L.la_prefill_workspace_size(4, 0, 16, 128, LA_BF16) == 0        # nothing to do
    assert L.la_prefill_workspace_size(256, 4096, 16, 128, LA_BF16) == 0       # enough CTAs: no segment split
    assert L.la_prefill_workspace_size(1, 100, 2, 96, LA_BF16) == 0        # unsupported D
    assert L.la_prefill_varlen_workspace_size(262144, 8, 16, 128, LA_BF16) > 0


# fake device pointers (aligned, never dereferenced: every case below fails in the host checks)
Q, K, V, O, S0, SN, WS = (0x10000000 * (i + 1) for i in range(7))


def _prefill(L, q=Q, k=K, v=V, o=O, B=1, N=256, H=2, D=128, dt=LA_BF16, s0=None, sn=None, ws=WS, wsb=1 << 30):
    return L.la_prefill(q, k, v, o, B, N, H, D, dt, s0, sn, None, ws, wsb, None)


@pytest.mark.parametrize("kwargs, status", [
    (dict(q=None), 1),                 # null input
    (dict(o=None), 1),                 # null output
    (dict(D=96), 2),                   # unsupported head dim
    (dict(D=32), 2),
    (dict(H=0), 1),
    (dict(B=0), 1),
    (dict(N=-1), 1),
    (dict(dt=7), 1),
    (dict(q=Q + 8), 1),                # misaligned
    (dict(s0=S0 + 4), 1),              # misaligned state
    (dict(o=Q + 64), 1),               # o overlaps q
    (dict(ws=None, N=4096), 3),        # missing workspace on the segmented path
    (dict(wsb=16, N=4096), 3),         # workspace too small
    (dict(ws=WS + 16, N=4096), 1),     # workspace misaligned
    (dict(B=1 << 20, N=1 << 12), 2),   # more than 2^31 elements
])
def test_prefill_rejects_bad_arguments(L, kwargs, status):
    assert _prefill(L, **kwargs) == status
    assert L.la_last_error().decode() != ""
    assert L.la_last_launch_count() == 0


def test_varlen_rejects_bad_arguments(L):
    f = L.la_prefill_varlen
    assert f(Q, K, V, O, None, 2, 100, 2, 128, LA_BF16, None, None, None, WS, 1 << 30, None) == 1   # no cu_seqlens
    assert f(Q, K, V, O, 0x1002, 2, 100, 2, 128, LA_BF16, None, None, None, WS, 1 << 30, None) == 1  # misaligned cu
    assert f(Q, K, V, O, 0x1000, 0, 100, 2, 128, LA_BF16, None, None, None, WS, 1 << 30, None) == 1  # nseq = 0
    assert f(Q, K, V, O, 0x1000, 2, -1, 2, 128, LA_BF16, None, None, None, WS, 1 << 30, None) == 1   # T < 0
    assert f(Q, K, V, O, 0x1000, 2, 100, 2, 80, LA_BF16, None, None, None, WS, 1 << 30, None) == 2   # D


def test_decode_rejects_bad_arguments(L):
    f = L.la_decode_step
    assert f(Q, K, V, O, None, 4, 2, 128, LA_BF16, None, None) == 1        # no state
    assert f(Q, K, V, O, S0, 0, 2, 128, LA_BF16, None, None) == 1          # B = 0
    assert f(Q, K, V, O, S0, 4, 2, 48, LA_BF16, None, None) == 2           # D
    assert f(Q, K, V, O, S0 + 8, 4, 2, 128, LA_BF16, None, None) == 1      # misaligned state
    assert f(Q, K, V, O, Q, 4, 2, 128, LA_BF16, None, None) == 1           # state overlaps q


class _FakeCuda:
    """Just enough of a CUDA tensor for the binding's argument checks (no device needed)."""

    def __init__(self, index, contiguous=True):
        self.is_cuda = True
        self.device = torch.device("cuda", index)
        self._contiguous = contiguous

    def is_contiguous(self):
        return self._contiguous


def test_binding_refuses_tensors_off_the_current_device(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    binding._need_cuda(_FakeCuda(0), None, _FakeCuda(0))                 # all on the current device
    with pytest.raises(ValueError, match="one CUDA device"):
        binding._need_cuda(_FakeCuda(0), _FakeCuda(1))
    with pytest.raises(ValueError, match="current CUDA device"):
        binding._need_cuda(_FakeCuda(1), _FakeCuda(1))
    with pytest.raises(ValueError, match="contiguous"):
        binding._need_cuda(_FakeCuda(0, contiguous=False))


class _FakeStream:
    def __init__(self, index):
        self.device = torch.device("cuda", index)
        self.cuda_stream = 0


def test_binding_refuses_a_stream_of_another_device(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    assert binding._stream(_FakeStream(0)).value is None       # the current device's stream handle passes
    with pytest.raises(ValueError, match="stream is on cuda:1"):
        binding._stream(_FakeStream(1))


def test_binding_checks_sizes_and_dtypes_of_every_tensor():
    """The library gets bare pointers: a tensor smaller than the call's sizes, or of another element type,
    would be read or written past its end. The binding refuses each such case before calling it (CPU tensors
    stand in: the size checks do not look at the device)."""
    B, N, H, D = 2, 8, 3, 64
    q = torch.zeros(B, N, H, D, dtype=torch.bfloat16)
    st = torch.zeros(B, H, D, D)
    ok = dict(same=(("k", q), ("v", q)), states=(("initial_state", st, B),), slopes=torch.zeros(H),
              outs=(("o", torch.zeros(B, N, H, D, dtype=torch.float16)),), out_dtype=torch.float16)
    binding._check_sizes(q, **ok)
    bad = [
        dict(ok, same=(("k", q.float()),)),                                             # k of another dtype
        dict(ok, same=(("v", q[:, :4]),)),                                              # v shorter than q
        dict(ok, states=(("initial_state", st.half(), B),)),                            # fp16 state
        dict(ok, states=(("final_state", st[:1], B),)),                                 # state for one sequence
        dict(ok, states=(("state", torch.zeros(B, H, 128, 128), B),)),                  # state of the other D
        dict(ok, slopes=torch.zeros(H + 1)),                                            # slopes of H + 1 heads
        dict(ok, slopes=torch.zeros(H, dtype=torch.float64)),                           # fp64 slopes
        dict(ok, outs=(("o", torch.zeros(B, N - 1, H, D, dtype=torch.float16)),)),      # smaller o
        dict(ok, outs=(("o", torch.zeros(B, N, H, D, dtype=torch.float32)),)),          # o of another dtype
    ]
    for kw in bad:
        with pytest.raises(ValueError):
            binding._check_sizes(q, **kw)


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.la_prefill(x, x, x)


def test_plan_segments_of_at_least_two_chunks(L):
    # B=1, N=1024, H=16: 8 chunks over 16 heads would give one-chunk segments; the floor makes them two chunks,
    # so 4 segment-state slots (128 x 128 fp32 each per head) and the initial-state copies (64 KB per head)
    slot = 128 * 128 * 4
    assert L.la_prefill_workspace_size(1, 1024, 16, 128, LA_BF16) == (4 + 1) * 16 * slot
    # B=1, N=8192, H=2: two-chunk segments, and their state units are not split further (one-chunk units)
    assert L.la_prefill_workspace_size(1, 8192, 2, 128, LA_BF16) == (32 + 1) * 2 * slot
    # the corrected split (fp16 outputs): the same two-chunk floor; per segment and head an exit state and the
    # split image of its entry state (64 KB each), no copies of the initial state
    assert L.la_prefill_workspace_size(1, 1024, 16, 128, LA_BF16_F16OUT) == 2 * 4 * 16 * slot
    assert L.la_prefill_workspace_size(1, 8192, 2, 128, LA_BF16_F16OUT) == 2 * 32 * 2 * slot
    # a 256-token sequence is one segment of its two chunks: no split, no workspace
    assert L.la_prefill_workspace_size(1, 256, 16, 128, LA_BF16) == 0


def test_shard_state_workspace_size(L):
    # 64 chunks over at most 148 / 16 = 9 units: units of 8 chunks, 8 of them
    assert L.la_shard_state_workspace_size(1, 8192, 16, 128, LA_BF16) == 8 * 16 * 128 * 128 * 4
    assert L.la_shard_state_workspace_size(64, 4096, 16, 128, LA_BF16) == 0   # enough CTAs: one unit per sequence
    assert L.la_shard_state_workspace_size(1, 8192, 16, 128, LA_FP32) == 0    # tensor-core path only
    assert L.la_shard_state_workspace_size(1, 8192, 16, 64, LA_BF16) == 8 * 16 * 64 * 64 * 4   # D = 64: 64 x 64 units
    assert L.la_shard_state_workspace_size(1, 8192, 16, 96, LA_BF16) == 0     # unsupported D


def test_shard_state_rejects_bad_arguments(L):
    f = L.la_shard_state
    assert f(K, V, 1, 256, 2, 128, LA_FP32, None, S0, WS, 1 << 30, None) == 2       # fp32 inputs
    assert f(K, V, 1, 256, 2, 96, LA_BF16, None, S0, WS, 1 << 30, None) == 2        # D
    assert f(K, V, 0, 256, 2, 128, LA_BF16, None, S0, WS, 1 << 30, None) == 1       # B
    assert f(K, V, 1, 256, 2, 128, LA_BF16, None, None, WS, 1 << 30, None) == 1     # no output
    assert f(K, V, 1, 256, 2, 128, LA_BF16, None, S0 + 4, WS, 1 << 30, None) == 1   # misaligned output
    assert f(None, V, 1, 256, 2, 128, LA_BF16, None, S0, WS, 1 << 30, None) == 1    # no k
    assert f(K, V, 1, 8192, 16, 128, LA_BF16, None, S0, None, 0, None) == 3         # workspace missing
    assert L.la_last_launch_count() == 0


def test_cp_entry_state_rejects_bad_arguments(L):
    f = L.la_cp_entry_state
    assert f(WS, 4, 4, 1, 2, 128, 512, None, None, S0, None) == 1     # rank out of range
    assert f(WS, 4, -1, 1, 2, 128, 512, None, None, S0, None) == 1
    assert f(None, 4, 2, 1, 2, 128, 512, None, None, S0, None) == 1   # rank > 0 needs the gathered states
    assert f(WS, 4, 1, 1, 2, 96, 512, None, None, S0, None) == 2      # D
    assert f(WS, 4, 1, 1, 2, 128, 512, None, None, None, None) == 1   # no output
    assert f(WS, 4, 1, 1, 2, 128, 512, None, None, WS + 64, None) == 1  # output overlaps the gathered states


# --------------------------------------------------------------------------- backward pass
def test_backward_workspace_size(L):
    # two transposed-state slots, then three sweep slots. 64 (sequence, head) pairs: two unsegmented sweeps
    # fill the GPU but three would not, so the dv sweep runs first with the whole GPU's segmented plan (reversed
    # in time: at least the forward prefill's segment states) and the dq and dk sweeps then run unsegmented
    slot = 4 * 16 * 128 * 128 * 4
    fwd = L.la_prefill_workspace_size(4, 4096, 16, 128, LA_BF16)
    assert fwd > 0
    ws = L.la_prefill_backward_workspace_size(4, 4096, 16, 128, LA_BF16)
    assert ws >= 2 * slot + 3 * fwd and (ws - 2 * slot) % 3 == 0
    # 128 pairs: all three sweeps at once, unsegmented, no sweep workspace
    slot8 = 8 * 16 * 128 * 128 * 4
    assert L.la_prefill_backward_workspace_size(8, 4096, 16, 128, LA_BF16) == 2 * slot8
    # one long sequence of two heads is still cut into segments, whose states need room
    slot1 = 2 * 128 * 128 * 4
    ws1 = L.la_prefill_backward_workspace_size(1, 65536, 2, 128, LA_BF16)
    assert ws1 >= 2 * slot1 + 3 * 2 * 128 * 128 * 4
    assert L.la_prefill_backward_workspace_size(4, 4096, 16, 128, LA_FP32) == 2 * slot   # no sweep workspace
    assert L.la_prefill_backward_workspace_size(1, 100, 2, 96, LA_BF16) == 0              # unsupported D
    assert L.la_prefill_varlen_backward_workspace_size(262144, 8, 16, 128, LA_BF16) > 0


DO, DQ, DK, DV = (0x90000000 + 0x10000000 * i for i in range(4))


def _backward(L, q=Q, k=K, v=V, do=DO, dq=DQ, dk=DK, dv=DV, B=1, N=256, H=2, D=128, dt=LA_BF16, s0=None, dsn=None,
              ds0=None, ws=WS, wsb=1 << 30):
    return L.la_prefill_backward(q, k, v, do, dq, dk, dv, B, N, H, D, dt, s0, dsn, ds0, None, ws, wsb, None)


@pytest.mark.parametrize("kwargs, status", [
    (dict(do=None), 1),                # null output gradient
    (dict(dk=None), 1),                # null gradient buffer
    (dict(dq=None), 1),
    (dict(D=96), 2),                   # unsupported head dim
    (dict(B=0), 1),
    (dict(dk=DQ + 64), 1),             # gradients overlap each other
    (dict(dv=DO + 64), 1),             # a gradient overlaps an input
    (dict(ds0=S0 + 4), 1),             # misaligned d_initial_state
    (dict(do=DO + 8), 1),              # misaligned dout
    (dict(ws=None), 3),                # the backward pass always needs a workspace
    (dict(wsb=64), 3),
    (dict(ws=WS + 16), 1),
])
def test_backward_rejects_bad_arguments(L, kwargs, status):
    assert _backward(L, **kwargs) == status
    assert L.la_last_error().decode() != ""
    assert L.la_last_launch_count() == 0


def test_varlen_backward_rejects_bad_arguments(L):
    f = L.la_prefill_varlen_backward
    assert f(Q, K, V, DO, DQ, DK, DV, None, 2, 100, 2, 128, LA_BF16, None, None, None, None, WS, 1 << 30, None) == 1
    assert f(Q, K, V, DO, DQ, DK, DV, 0x1002, 2, 100, 2, 128, LA_BF16, None, None, None, None, WS, 1 << 30,
             None) == 1
    assert f(Q, K, V, DO, DQ, DK, DV, 0x1000, 0, 100, 2, 128, LA_BF16, None, None, None, None, WS, 1 << 30,
             None) == 1


# --------------------------------------------------------------------------- fused output norm + gate
def test_norm_gate_rejects_bad_arguments(L):
    f = L.la_prefill_norm_gate
    G, NW = 0x50000000, 0x51000000
    args = lambda g=G, w=NW, eps=1e-6, o=O: (Q, K, V, g, w, eps, o, 1, 256, 2, 128, LA_BF16, None, None, None, WS,  # noqa: E731
                                           1 << 30, None)
    assert f(*args(g=None)) == 1            # no gate
    assert f(*args(w=None)) == 1            # no weight
    assert f(*args(g=G + 8)) == 1           # misaligned gate
    assert f(*args(eps=-1.0)) == 1          # negative eps
    assert f(*args(eps=float("nan"))) == 1
    assert f(*args(o=G + 64)) == 1          # o overlaps the gate
    assert L.la_last_launch_count() == 0
    d = L.la_decode_steps_norm_gate
    assert d(Q, K, V, None, NW, 1e-6, O, S0, 4, 2, 2, 128, LA_BF16, None, None) == 1


def test_norm_gate_alone_rejects_bad_arguments(L):
    f = L.la_norm_gate
    G, NW, Y = 0x50000000, 0x51000000, 0x52000000
    assert f(O, G, NW, 1e-6, Y, 100, 2, 96, LA_BF16, None) == 2      # D
    assert f(O, None, NW, 1e-6, Y, 100, 2, 128, LA_BF16, None) == 1   # no gate
    assert f(O, G, NW, -1.0, Y, 100, 2, 128, LA_BF16, None) == 1      # eps
    assert f(O, G, NW, 1e-6, O + 256, 100, 2, 128, LA_BF16, None) == 1  # y partly overlaps o
    assert f(O, G, NW, 1e-6, G, 100, 2, 128, LA_BF16, None) == 1      # y overlaps the gate
    assert f(O + 8, G, NW, 1e-6, Y, 100, 2, 128, LA_BF16, None) == 1  # misaligned o
    assert L.la_last_launch_count() == 0


def test_cp_backward_calls_reject_bad_arguments(L):
    f = L.la_shard_state_reverse
    assert f(Q, DO, 1, 256, 2, 128, LA_FP32, None, S0, WS, 1 << 30, None) == 2       # fp32 inputs
    assert f(Q, DO, 1, 256, 2, 96, LA_BF16, None, S0, WS, 1 << 30, None) == 2        # D
    assert f(Q, DO, 1, 256, 2, 128, LA_BF16, None, None, WS, 1 << 30, None) == 1     # no output
    assert f(None, DO, 1, 256, 2, 128, LA_BF16, None, S0, WS, 1 << 30, None) == 1    # no q
    assert f(Q, DO, 1, 8192, 16, 128, LA_BF16, None, S0, None, 0, None) == 3         # workspace missing
    e = L.la_cp_reverse_entry_state
    assert e(WS, 4, 4, 1, 2, 128, 512, None, None, S0, None) == 1     # rank out of range
    assert e(None, 4, 1, 1, 2, 128, 512, None, None, S0, None) == 1   # not the last rank: needs the gathered states
    assert e(WS, 4, 1, 1, 2, 96, 512, None, None, S0, None) == 2      # D
    assert e(WS, 4, 1, 1, 2, 128, 512, None, None, WS + 64, None) == 1  # output overlaps the gathered states
    assert L.la_last_launch_count() == 0


def test_varlen_cp_entry_states_reject_bad_arguments(L):
    """The host checks of the varlen context-parallel entry states (cu_seqlens is a host array here): every case
    fails before anything touches CUDA."""
    cu_t = ctypes.c_int32 * 4
    good = cu_t(0, 100, 100, 300)       # T = 300
    G, S0, OUT = 0x10000000, 0x20000000, 0x30000000
    # shards of 100 tokens: sequence 2 ([100, 300)) enters rank 2 from rank 1 and leaves rank 1 for rank 2, so the
    # forward entry state of rank 2 and the reversed one of rank 1 need the gathered states
    for f, needy in ((L.la_cp_varlen_entry_state, 2), (L.la_cp_varlen_reverse_entry_state, 1)):
        call = lambda g=G, R=3, rank=needy, cu=good, nseq=3, H=2, D=128, s=S0, out=OUT: f(  # noqa: E731
            g, R, rank, cu, nseq, H, D, s, None, out, None)
        assert call(cu=None) == 1                      # no cu_seqlens
        assert call(cu=cu_t(1, 100, 100, 300)) == 1    # cu[0] != 0
        assert call(cu=cu_t(0, 100, 90, 300)) == 1     # decreasing
        assert call(R=7) == 1                          # T = 300 not divisible by 7
        assert call(R=100, rank=0, cu=cu_t(0, 100, 100, 300)) == 2   # more ranks than supported
        assert call(rank=3) == 1 and call(rank=-1) == 1
        assert call(nseq=0) == 1
        assert call(D=96) == 2
        assert call(H=0) == 1
        assert call(out=None) == 1 and call(out=OUT + 4) == 1
        assert call(s=S0 + 8) == 1                     # misaligned given state
        assert call(g=None) == 1                       # the crossing sequence needs the other ranks' states
        assert call(out=G) == 1                        # output overlaps gathered


def test_static_scratch_covers_every_uniform_plan(L):
    """la_prefill_noalloc serves every uniform batch the library plans: over a sweep of shapes, the workspace
    la_prefill needs stays within the fixed LA_STATIC_WORKSPACE_BYTES (the segment split stops at about one
    unit per SM, each unit and head holding one 64 KiB state, or with the corrected split of fp16 / fp32
    outputs an exit state and an entry-state image)."""
    limit = 32 << 20
    worst = 0
    for D in (64, 128):
        for B in (1, 2, 3, 4, 8, 16, 37, 74, 148):
            for H in (1, 2, 4, 8, 16, 32, 64):
                for N in (1, 127, 128, 1000, 4096, 65536, 1 << 20):
                    if B * N * H * D >= 1 << 31:
                        continue
                    for dt in (LA_BF16, LA_BF16_F16OUT, LA_BF16_F32OUT):
                        worst = max(worst, L.la_prefill_workspace_size(B, N, H, D, dt))
    assert 0 < worst <= limit, worst
