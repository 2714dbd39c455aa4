"""Thin ctypes binding of the C ABI in include/la.h, with the same names.

Only argument marshalling happens here: torch tensors supply device memory
and the current CUDA stream; every step of the operator runs in the library's
kernels. There is no fallback: if the library or a GPU is missing, every call
raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libla_b200.so")

LA_OK, LA_ERR_INVALID_ARGUMENT, LA_ERR_UNSUPPORTED, LA_ERR_WORKSPACE, LA_ERR_CUDA, LA_ERR_DEVICE_TIMEOUT = range(6)
LA_BF16, LA_FP32, LA_BF16_F32OUT, LA_BF16_F16OUT = 0, 1, 2, 3

# Every symbol include/la.h declares.
EXPORTS = (
    "la_prefill_workspace_size", "la_prefill", "la_prefill_varlen_workspace_size", "la_prefill_varlen",
    "la_decode_step", "la_status_string", "la_last_error", "la_validate_cu_seqlens", "la_get_device_error",
    "la_last_launch_count", "la_trace_enable", "la_trace_collect", "la_prefill_noalloc",
    "la_shard_state_workspace_size", "la_shard_state", "la_cp_entry_state", "la_decode_steps",
    "la_prefill_backward_workspace_size", "la_prefill_backward", "la_prefill_varlen_backward_workspace_size",
    "la_prefill_varlen_backward", "la_prefill_norm_gate", "la_prefill_varlen_norm_gate", "la_decode_steps_norm_gate",
    "la_norm_gate", "la_shard_state_reverse", "la_cp_reverse_entry_state", "la_cp_varlen_entry_state",
    "la_cp_varlen_reverse_entry_state",
)


class LAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


_lib = None


def lib():
    """Load libla_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                              "(run linear_attention_hybrid_b200.build.build())")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, i64, f = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64, ctypes.c_int
        L.la_prefill_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.la_prefill_workspace_size.restype = sz
        L.la_prefill.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        L.la_prefill.restype = f
        L.la_prefill_varlen_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        L.la_prefill_varlen_workspace_size.restype = sz
        L.la_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        L.la_prefill_varlen.restype = f
        L.la_decode_step.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp]
        L.la_decode_step.restype = f
        L.la_status_string.argtypes = [f]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_last_error.argtypes = []
        L.la_last_error.restype = ctypes.c_char_p
        L.la_validate_cu_seqlens.argtypes = [vp, i32, i64, vp]
        L.la_validate_cu_seqlens.restype = f
        L.la_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.la_get_device_error.restype = f
        L.la_last_launch_count.argtypes = []
        L.la_last_launch_count.restype = ctypes.c_int
        L.la_trace_enable.argtypes = [i32]
        L.la_trace_enable.restype = f
        L.la_trace_collect.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float), i32]
        L.la_trace_collect.restype = ctypes.c_int
        L.la_prefill_noalloc.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.la_prefill_noalloc.restype = f
        L.la_shard_state_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.la_shard_state_workspace_size.restype = sz
        L.la_shard_state.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        L.la_shard_state.restype = f
        L.la_cp_entry_state.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.la_cp_entry_state.restype = f
        L.la_decode_steps.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
        L.la_decode_steps.restype = f
        L.la_prefill_backward_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.la_prefill_backward_workspace_size.restype = sz
        L.la_prefill_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz,
                                          vp]
        L.la_prefill_backward.restype = f
        L.la_prefill_varlen_backward_workspace_size.argtypes = [i64, i32, i32, i32, i32]
        L.la_prefill_varlen_backward_workspace_size.restype = sz
        L.la_prefill_varlen_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp,
                                                 vp, vp, sz, vp]
        L.la_prefill_varlen_backward.restype = f
        fl = ctypes.c_float
        L.la_prefill_norm_gate.argtypes = [vp, vp, vp, vp, vp, fl, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, sz, vp]
        L.la_prefill_norm_gate.restype = f
        L.la_prefill_varlen_norm_gate.argtypes = [vp, vp, vp, vp, vp, fl, vp, vp, i32, i64, i32, i32, i32, vp, vp, vp,
                                                  vp, sz, vp]
        L.la_prefill_varlen_norm_gate.restype = f
        L.la_decode_steps_norm_gate.argtypes = [vp, vp, vp, vp, vp, fl, vp, vp, i32, i32, i32, i32, i32, vp, vp]
        L.la_decode_steps_norm_gate.restype = f
        L.la_norm_gate.argtypes = [vp, vp, vp, fl, vp, i64, i32, i32, i32, vp]
        L.la_norm_gate.restype = f
        L.la_shard_state_reverse.argtypes = [vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, sz, vp]
        L.la_shard_state_reverse.restype = f
        L.la_cp_reverse_entry_state.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp]
        L.la_cp_reverse_entry_state.restype = f
        L.la_cp_varlen_entry_state.argtypes = [vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp]
        L.la_cp_varlen_entry_state.restype = f
        L.la_cp_varlen_reverse_entry_state.argtypes = [vp, i32, i32, vp, i32, i32, i32, vp, vp, vp, vp]
        L.la_cp_varlen_reverse_entry_state.restype = f
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != LA_OK:
        L = lib()
        raise LAError(status, f"{what}: {L.la_status_string(status).decode()}: {L.la_last_error().decode()}")


def _code_of(in_dtype, out_dtype=None) -> int:
    """la_dtype for inputs of in_dtype and an output of out_dtype (default: the input dtype)."""
    out_dtype = in_dtype if out_dtype is None else out_dtype
    if in_dtype == torch.bfloat16 and out_dtype == torch.bfloat16:
        return LA_BF16
    if in_dtype == torch.bfloat16 and out_dtype == torch.float32:
        return LA_BF16_F32OUT
    if in_dtype == torch.bfloat16 and out_dtype == torch.float16:
        return LA_BF16_F16OUT
    if in_dtype == torch.float32 and out_dtype == torch.float32:
        return LA_FP32
    raise TypeError(f"unsupported dtypes: inputs {in_dtype}, output {out_dtype}")


def _dtype_code(t: torch.Tensor, out_dtype=None) -> int:
    return _code_of(t.dtype, out_dtype)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    """The stream handle to launch on: the current stream, or `stream`, which must belong to the current device
    (the library launches on the current device; a stream of another device fails inside the launch)."""
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device.index != torch.cuda.current_device():
        raise ValueError(f"the stream is on {stream.device} but the current CUDA device is "
                         f"cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    """Every tensor a CUDA tensor, contiguous, and on the current device (the library launches on the current
    device and its current stream; memory of another device would be read through an invalid address)."""
    dev = None
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("all tensors must be CUDA tensors (there is no CPU path)")
            if not t.is_contiguous():
                raise ValueError("all tensors must be contiguous")
            if dev is None:
                dev = t.device
            elif t.device != dev:
                raise ValueError(f"all tensors must be on one CUDA device (got {dev} and {t.device})")
    if dev is not None and dev.index != torch.cuda.current_device():
        raise ValueError(f"the tensors are on {dev} but the current CUDA device is cuda:{torch.cuda.current_device()}; "
                         f"call under torch.cuda.device({dev.index})")


def _check_sizes(ref, same=(), states=(), slopes=None, outs=(), out_dtype=None, H=None, D=None):
    """Shapes and dtypes of every tensor a call hands the library. The C ABI receives bare pointers, so this is
    the one place where a tensor of the wrong size or element type can be caught before a kernel reads or
    writes past its end.
      ref    : the tensor whose shape and dtype `same` and `outs` must have (q, or o for la_norm_gate)
      same   : (name, tensor) inputs with ref's shape and dtype (k, v, the gate, dout)
      states : (name, tensor, leading) fp32 states [leading, H, D, D]
      slopes : fp32 with H elements
      outs   : (name, tensor) outputs with ref's shape and dtype out_dtype
    Tensors given as None are skipped."""
    H = ref.shape[-2] if H is None else H
    D = ref.shape[-1] if D is None else D
    for name, t in same:
        if t is not None and (tuple(t.shape) != tuple(ref.shape) or t.dtype != ref.dtype):
            raise ValueError(f"{name} must have shape {tuple(ref.shape)} and dtype {ref.dtype} "
                             f"(got {tuple(t.shape)}, {t.dtype})")
    for name, t, lead in states:
        if t is not None and (tuple(t.shape) != (lead, H, D, D) or t.dtype != torch.float32):
            raise ValueError(f"{name} must be float32 of shape {(lead, H, D, D)} (got {tuple(t.shape)}, {t.dtype})")
    if slopes is not None and (slopes.dtype != torch.float32 or slopes.numel() != H):
        raise ValueError(f"slopes must be float32 with H={H} elements (got {slopes.numel()}, {slopes.dtype})")
    for name, t in outs:
        if t is not None and (tuple(t.shape) != tuple(ref.shape) or t.dtype != out_dtype):
            raise ValueError(f"{name} must have shape {tuple(ref.shape)} and dtype {out_dtype} "
                             f"(got {tuple(t.shape)}, {t.dtype})")


def la_status_string(status: int) -> str:
    return lib().la_status_string(status).decode()


def la_last_error() -> str:
    return lib().la_last_error().decode()


def la_last_launch_count() -> int:
    return int(lib().la_last_launch_count())


def la_trace_enable(on: bool = True) -> None:
    """Record CUDA events around every kernel later calls on this thread enqueue."""
    _check(lib().la_trace_enable(1 if on else 0), "la_trace_enable")


def la_trace_collect(max_entries: int = 4096):
    """Wait for the recorded kernels; return [(kernel name, milliseconds)] in launch order and clear."""
    names = (ctypes.c_char_p * max_entries)()
    ms = (ctypes.c_float * max_entries)()
    n = lib().la_trace_collect(names, ms, max_entries)
    if n < 0:
        raise LAError(LA_ERR_CUDA, "la_trace_collect: CUDA error while reading events")
    return [(names[i].decode(), float(ms[i])) for i in range(n)]


def la_prefill_workspace_size(B: int, N: int, H: int, D: int, dtype=torch.bfloat16, out_dtype=None) -> int:
    """Workspace bytes for la_prefill with inputs of `dtype` and outputs of `out_dtype` (default: `dtype`);
    the work split, and with it the size, depends on both."""
    return int(lib().la_prefill_workspace_size(B, N, H, D, _code_of(dtype, out_dtype)))


def la_prefill_varlen_workspace_size(T: int, nseq: int, H: int, D: int, dtype=torch.bfloat16, out_dtype=None) -> int:
    return int(lib().la_prefill_varlen_workspace_size(T, nseq, H, D, _code_of(dtype, out_dtype)))


def _workspace(nbytes: int, device, workspace):
    if nbytes == 0:
        return None
    if workspace is not None:
        if workspace.numel() * workspace.element_size() < nbytes:
            raise ValueError(f"workspace needs {nbytes} bytes")
        return workspace
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def la_prefill(q, k, v, initial_state=None, final_state=None, return_final_state=False, slopes=None, o=None,
               workspace=None, stream=None, out_dtype=None):
    """Chunked prefill. q, k, v: [B, N, H, D] (bf16 or fp32); o in out_dtype (default: q's dtype; bf16
    inputs may ask for fp32 o). Returns o, or (o, final_state) when return_final_state is set or a
    final_state buffer is given (it may be initial_state itself)."""
    _need_cuda(q, k, v, initial_state, final_state, slopes, o, workspace)
    B, N, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, N, H, D]")
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v)), states=(("initial_state", initial_state, B), ("final_state", final_state, B)),
                 slopes=slopes, outs=(("o", o),), out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    ws = _workspace(la_prefill_workspace_size(B, N, H, D, q.dtype, out_dtype), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, N, H, D, dt, _ptr(initial_state), _ptr(final_state),
                          _ptr(slopes), _ptr(ws), nb, _stream(stream))
    _check(st, "la_prefill")
    return (o, final_state) if final_state is not None else o


def la_prefill_noalloc(q, k, v, initial_state=None, final_state=None, return_final_state=False, slopes=None,
                       o=None, stream=None, out_dtype=None):
    """la_prefill for callers that cannot allocate device scratch: the library uses a fixed scratch array
    of its own (LA_STATIC_WORKSPACE_BYTES per GPU) instead of a workspace argument. The output and the
    final state are still the caller's buffers (allocated here only when not given). Calls that overlap
    on the GPU share that array and race; order them on one stream."""
    _need_cuda(q, k, v, initial_state, final_state, slopes, o)
    B, N, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, N, H, D]")
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v)), states=(("initial_state", initial_state, B), ("final_state", final_state, B)),
                 slopes=slopes, outs=(("o", o),), out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    st = lib().la_prefill_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, N, H, D, dt, _ptr(initial_state),
                                  _ptr(final_state), _ptr(slopes), _stream(stream))
    _check(st, "la_prefill_noalloc")
    return (o, final_state) if final_state is not None else o


def la_prefill_varlen(q, k, v, cu_seqlens, initial_state=None, final_state=None, return_final_state=False,
                      slopes=None, o=None, workspace=None, stream=None, out_dtype=None):
    """Packed varlen prefill. q, k, v: [T, H, D]; cu_seqlens: int32 CUDA tensor [nseq + 1]; o as in la_prefill."""
    _need_cuda(q, k, v, cu_seqlens, initial_state, final_state, slopes, o, workspace)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    T, H, D = q.shape
    nseq = cu_seqlens.numel() - 1
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v)),
                 states=(("initial_state", initial_state, nseq), ("final_state", final_state, nseq)),
                 slopes=slopes, outs=(("o", o),), out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((nseq, H, D, D), dtype=torch.float32, device=q.device)
    ws = _workspace(la_prefill_varlen_workspace_size(T, nseq, H, D, q.dtype, out_dtype), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(cu_seqlens), nseq, T, H, D, dt,
                                 _ptr(initial_state), _ptr(final_state), _ptr(slopes), _ptr(ws), nb, _stream(stream))
    _check(st, "la_prefill_varlen")
    return (o, final_state) if final_state is not None else o


def la_decode_step(q, k, v, state, slopes=None, o=None, stream=None, out_dtype=None):
    """One decode step, state [B, H, D, D] fp32 updated in place. q, k, v: [B, H, D]. Returns o."""
    _need_cuda(q, k, v, state, slopes, o)
    B, H, D = q.shape
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v)), states=(("state", state, B),), slopes=slopes, outs=(("o", o),),
                 out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    st = lib().la_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state), B, H, D, dt, _ptr(slopes),
                              _stream(stream))
    _check(st, "la_decode_step")
    return o


def la_decode_steps(q, k, v, state, slopes=None, o=None, stream=None, out_dtype=None):
    """K consecutive decode steps in one launch, state [B, H, D, D] fp32 updated in place (read and written
    once). q, k, v: [B, K, H, D]. Returns o [B, K, H, D]."""
    _need_cuda(q, k, v, state, slopes, o)
    B, K, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, K, H, D]")
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v)), states=(("state", state, B),), slopes=slopes, outs=(("o", o),),
                 out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    st = lib().la_decode_steps(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state), B, K, H, D, dt, _ptr(slopes),
                               _stream(stream))
    _check(st, "la_decode_steps")
    return o


# --------------------------------------------------------------------------- fused output norm + gate
def _norm_gate_args(q, gate, norm_weight, H, D):
    if gate.shape != q.shape or gate.dtype != q.dtype:
        raise ValueError("gate must have q's shape and dtype")
    if tuple(norm_weight.shape) != (H, D) or norm_weight.dtype != torch.float32:
        raise ValueError("norm_weight must be fp32 [H, D]")


def la_norm_gate(o, gate, norm_weight, eps=1e-6, y=None, stream=None):
    """y = norm_weight[h] * o / sqrt(mean over D of o^2 + eps) * sigmoid(gate) per (token, head), one streaming
    pass. o: [..., H, D] in the output dtype (bf16, fp16 or fp32); gate: same shape in the input dtype (bf16, or
    fp32 with an fp32 o); norm_weight [H, D] fp32. y defaults to a new tensor; pass y=o for in place."""
    _need_cuda(o, gate, norm_weight, y)
    H, D = o.shape[-2], o.shape[-1]
    if gate.shape != o.shape:
        raise ValueError("gate must have o's shape")
    if tuple(norm_weight.shape) != (H, D) or norm_weight.dtype != torch.float32:
        raise ValueError("norm_weight must be fp32 [H, D]")
    dt = _dtype_code(gate, o.dtype)
    _check_sizes(o, outs=(("y", y),), out_dtype=o.dtype)
    if y is None:
        y = torch.empty_like(o)
    T = o.numel() // (H * D)
    _check(lib().la_norm_gate(_ptr(o), _ptr(gate), _ptr(norm_weight), float(eps), _ptr(y), T, H, D, dt,
                              _stream(stream)), "la_norm_gate")
    return y


def la_prefill_norm_gate(q, k, v, gate, norm_weight, eps=1e-6, initial_state=None, final_state=None,
                         return_final_state=False, slopes=None, o=None, workspace=None, stream=None, out_dtype=None):
    """la_prefill followed by la_norm_gate in place:
    y = norm_weight[h] * o / sqrt(mean over D of o^2 + eps) * sigmoid(gate) per (token, head).
    gate: like q (bf16); norm_weight: [H, D] fp32. Returns y (and the final state) as la_prefill."""
    _need_cuda(q, k, v, gate, norm_weight, initial_state, final_state, slopes, o, workspace)
    B, N, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, N, H, D]")
    _norm_gate_args(q, gate, norm_weight, H, D)
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v), ("gate", gate)),
                 states=(("initial_state", initial_state, B), ("final_state", final_state, B)),
                 slopes=slopes, outs=(("o", o),), out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    ws = _workspace(la_prefill_workspace_size(B, N, H, D, q.dtype, out_dtype), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_prefill_norm_gate(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(norm_weight), float(eps), _ptr(o),
                                    B, N, H, D, dt, _ptr(initial_state), _ptr(final_state), _ptr(slopes), _ptr(ws),
                                    nb, _stream(stream))
    _check(st, "la_prefill_norm_gate")
    return (o, final_state) if final_state is not None else o


def la_prefill_varlen_norm_gate(q, k, v, gate, norm_weight, cu_seqlens, eps=1e-6, initial_state=None,
                                final_state=None, return_final_state=False, slopes=None, o=None, workspace=None,
                                stream=None, out_dtype=None):
    """la_prefill_varlen followed by la_norm_gate in place (gate [T, H, D])."""
    _need_cuda(q, k, v, gate, norm_weight, cu_seqlens, initial_state, final_state, slopes, o, workspace)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    T, H, D = q.shape
    _norm_gate_args(q, gate, norm_weight, H, D)
    nseq = cu_seqlens.numel() - 1
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v), ("gate", gate)),
                 states=(("initial_state", initial_state, nseq), ("final_state", final_state, nseq)),
                 slopes=slopes, outs=(("o", o),), out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if final_state is None and return_final_state:
        final_state = torch.empty((nseq, H, D, D), dtype=torch.float32, device=q.device)
    ws = _workspace(la_prefill_varlen_workspace_size(T, nseq, H, D, q.dtype, out_dtype), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_prefill_varlen_norm_gate(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(norm_weight), float(eps),
                                           _ptr(o), _ptr(cu_seqlens), nseq, T, H, D, dt, _ptr(initial_state),
                                           _ptr(final_state), _ptr(slopes), _ptr(ws), nb, _stream(stream))
    _check(st, "la_prefill_varlen_norm_gate")
    return (o, final_state) if final_state is not None else o


def la_decode_steps_norm_gate(q, k, v, gate, norm_weight, state, eps=1e-6, slopes=None, o=None, stream=None,
                              out_dtype=None):
    """la_decode_steps with the output norm + gate fused into the decode kernel. q, k, v, gate: [B, K, H, D];
    state updated in place."""
    _need_cuda(q, k, v, gate, norm_weight, state, slopes, o)
    B, K, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must have the same shape [B, K, H, D]")
    _norm_gate_args(q, gate, norm_weight, H, D)
    if o is not None and out_dtype is None:
        out_dtype = o.dtype
    dt = _dtype_code(q, out_dtype)
    _check_sizes(q, same=(("k", k), ("v", v), ("gate", gate)), states=(("state", state, B),), slopes=slopes,
                 outs=(("o", o),), out_dtype=out_dtype or q.dtype)
    if o is None:
        o = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    st = lib().la_decode_steps_norm_gate(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(norm_weight), float(eps),
                                         _ptr(o), _ptr(state), B, K, H, D, dt, _ptr(slopes), _stream(stream))
    _check(st, "la_decode_steps_norm_gate")
    return o


# --------------------------------------------------------------------------- backward pass
def la_prefill_backward_workspace_size(B: int, N: int, H: int, D: int, dtype=torch.bfloat16) -> int:
    code = LA_BF16 if dtype == torch.bfloat16 else LA_FP32
    return int(lib().la_prefill_backward_workspace_size(B, N, H, D, code))


def la_prefill_varlen_backward_workspace_size(T: int, nseq: int, H: int, D: int, dtype=torch.bfloat16) -> int:
    code = LA_BF16 if dtype == torch.bfloat16 else LA_FP32
    return int(lib().la_prefill_varlen_backward_workspace_size(T, nseq, H, D, code))


def _grads(q, dq, dk, dv, out_dtype):
    if dq is not None and out_dtype is None:
        out_dtype = dq.dtype
    out_dtype = out_dtype or q.dtype
    dq, dk, dv = (torch.empty(q.shape, dtype=out_dtype, device=q.device) if g is None else g for g in (dq, dk, dv))
    return dq, dk, dv, out_dtype


def la_prefill_backward(q, k, v, dout, initial_state=None, d_final_state=None, d_initial_state=None,
                        return_d_initial_state=False, slopes=None, dq=None, dk=None, dv=None, workspace=None,
                        stream=None, out_dtype=None):
    """Gradients of la_prefill: q, k, v, dout [B, N, H, D] (bf16 or fp32); dq, dk, dv in out_dtype (default:
    q's dtype). initial_state is the forward's S0 and d_final_state the gradient of its final state (both
    [B, H, D, D] fp32 or None). Returns (dq, dk, dv), plus d_initial_state when asked for or given."""
    _need_cuda(q, k, v, dout, initial_state, d_final_state, d_initial_state, slopes, dq, dk, dv, workspace)
    B, N, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or dout.shape != q.shape or dout.dtype != q.dtype:
        raise ValueError("q, k, v and dout must have the same shape [B, N, H, D] and dtype")
    dq, dk, dv, out_dtype = _grads(q, dq, dk, dv, out_dtype)
    dt = _dtype_code(q, out_dtype)
    if d_initial_state is None and return_d_initial_state:
        d_initial_state = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    _check_sizes(q, same=(("k", k), ("v", v), ("dout", dout)),
                 states=(("initial_state", initial_state, B), ("d_final_state", d_final_state, B),
                         ("d_initial_state", d_initial_state, B)),
                 slopes=slopes, outs=(("dq", dq), ("dk", dk), ("dv", dv)), out_dtype=out_dtype)
    ws = _workspace(la_prefill_backward_workspace_size(B, N, H, D, q.dtype), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), B, N, H, D,
                                   dt, _ptr(initial_state), _ptr(d_final_state), _ptr(d_initial_state), _ptr(slopes),
                                   _ptr(ws), nb, _stream(stream))
    _check(st, "la_prefill_backward")
    return (dq, dk, dv, d_initial_state) if d_initial_state is not None else (dq, dk, dv)


def la_prefill_varlen_backward(q, k, v, dout, cu_seqlens, initial_state=None, d_final_state=None,
                               d_initial_state=None, return_d_initial_state=False, slopes=None, dq=None, dk=None,
                               dv=None, workspace=None, stream=None, out_dtype=None):
    """Gradients of la_prefill_varlen: q, k, v, dout [T, H, D]; cu_seqlens int32 [nseq + 1]; states
    [nseq, H, D, D]. Returns as la_prefill_backward."""
    _need_cuda(q, k, v, dout, cu_seqlens, initial_state, d_final_state, d_initial_state, slopes, dq, dk, dv,
               workspace)
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    T, H, D = q.shape
    if k.shape != q.shape or v.shape != q.shape or dout.shape != q.shape or dout.dtype != q.dtype:
        raise ValueError("q, k, v and dout must have the same shape [T, H, D] and dtype")
    nseq = cu_seqlens.numel() - 1
    dq, dk, dv, out_dtype = _grads(q, dq, dk, dv, out_dtype)
    dt = _dtype_code(q, out_dtype)
    if d_initial_state is None and return_d_initial_state:
        d_initial_state = torch.empty((nseq, H, D, D), dtype=torch.float32, device=q.device)
    _check_sizes(q, same=(("k", k), ("v", v), ("dout", dout)),
                 states=(("initial_state", initial_state, nseq), ("d_final_state", d_final_state, nseq),
                         ("d_initial_state", d_initial_state, nseq)),
                 slopes=slopes, outs=(("dq", dq), ("dk", dk), ("dv", dv)), out_dtype=out_dtype)
    ws = _workspace(la_prefill_varlen_backward_workspace_size(T, nseq, H, D, q.dtype), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_prefill_varlen_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                          _ptr(cu_seqlens), nseq, T, H, D, dt, _ptr(initial_state),
                                          _ptr(d_final_state), _ptr(d_initial_state), _ptr(slopes), _ptr(ws), nb,
                                          _stream(stream))
    _check(st, "la_prefill_varlen_backward")
    return (dq, dk, dv, d_initial_state) if d_initial_state is not None else (dq, dk, dv)


def la_validate_cu_seqlens(cu_seqlens, T: int, stream=None) -> None:
    _check(lib().la_validate_cu_seqlens(_ptr(cu_seqlens), cu_seqlens.numel() - 1, T, _stream(stream)),
           "la_validate_cu_seqlens")


def la_get_device_error() -> int:
    """Synchronise, then read and clear the library's device status word (LA_OK if clean)."""
    code = ctypes.c_int(0)
    _check(lib().la_get_device_error(ctypes.byref(code)), "la_get_device_error")
    return code.value


# --------------------------------------------------------------------------- context parallelism
def la_shard_state_workspace_size(B: int, N: int, H: int, D: int) -> int:
    return int(lib().la_shard_state_workspace_size(B, N, H, D, LA_BF16))


def la_shard_state(k, v, slopes=None, delta_state=None, workspace=None, stream=None):
    """State a shard produces from a zero start: dS = sum_s lambda^(N-1-s) k_s^T v_s per sequence and head.
    k, v: [B, N, H, D] bf16, D = 64 or 128. Returns delta_state [B, H, D, D] fp32."""
    _need_cuda(k, v, slopes, delta_state, workspace)
    B, N, H, D = k.shape
    if v.shape != k.shape:
        raise ValueError("k and v must have the same shape [B, N, H, D]")
    if k.dtype != torch.bfloat16:
        raise TypeError("la_shard_state takes bf16 k and v")
    _check_sizes(k, same=(("v", v),), states=(("delta_state", delta_state, B),), slopes=slopes)
    if delta_state is None:
        delta_state = torch.empty((B, H, D, D), dtype=torch.float32, device=k.device)
    ws = _workspace(la_shard_state_workspace_size(B, N, H, D), k.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_shard_state(_ptr(k), _ptr(v), B, N, H, D, LA_BF16, _ptr(slopes), _ptr(delta_state), _ptr(ws), nb,
                              _stream(stream))
    _check(st, "la_shard_state")
    return delta_state


def la_cp_entry_state(gathered, rank: int, L: int, initial_state=None, slopes=None, s_in=None, stream=None):
    """State entering shard `rank` of a context-parallel group: gathered [R, B, H, D, D] holds every
    shard's la_shard_state in rank order, L is the tokens per shard. Returns s_in [B, H, D, D] fp32."""
    _need_cuda(gathered, initial_state, slopes, s_in)
    R, B, H, D, _ = gathered.shape
    if gathered.dtype != torch.float32 or tuple(gathered.shape) != (R, B, H, D, D):
        raise ValueError(f"gathered must be float32 [R, B, H, D, D] (got {tuple(gathered.shape)}, {gathered.dtype})")
    _check_sizes(gathered, states=(("initial_state", initial_state, B), ("s_in", s_in, B)), slopes=slopes, H=H, D=D)
    if s_in is None:
        s_in = torch.empty((B, H, D, D), dtype=torch.float32, device=gathered.device)
    st = lib().la_cp_entry_state(_ptr(gathered), R, rank, B, H, D, L, _ptr(initial_state), _ptr(slopes), _ptr(s_in),
                                 _stream(stream))
    _check(st, "la_cp_entry_state")
    return s_in


def la_shard_state_reverse(q, dout, slopes=None, delta_state=None, workspace=None, stream=None):
    """Reversed state a shard produces from a zero start (the backward pass's sweep from the right):
    dH = sum_s lambda^(s+1) q_s^T dO_s per sequence and head, s from the shard's start. q, dout: [B, N, H, D]
    bf16, D = 64 or 128. Returns delta_state [B, H, D, D] fp32."""
    _need_cuda(q, dout, slopes, delta_state, workspace)
    B, N, H, D = q.shape
    if dout.shape != q.shape:
        raise ValueError("q and dout must have the same shape [B, N, H, D]")
    if q.dtype != torch.bfloat16 or dout.dtype != torch.bfloat16:
        raise TypeError("la_shard_state_reverse takes bf16 q and dout")
    _check_sizes(q, same=(("dout", dout),), states=(("delta_state", delta_state, B),), slopes=slopes)
    if delta_state is None:
        delta_state = torch.empty((B, H, D, D), dtype=torch.float32, device=q.device)
    ws = _workspace(la_shard_state_workspace_size(B, N, H, D), q.device, workspace)
    nb = 0 if ws is None else ws.numel() * ws.element_size()
    st = lib().la_shard_state_reverse(_ptr(q), _ptr(dout), B, N, H, D, LA_BF16, _ptr(slopes), _ptr(delta_state),
                                      _ptr(ws), nb, _stream(stream))
    _check(st, "la_shard_state_reverse")
    return delta_state


def la_cp_reverse_entry_state(gathered, rank: int, L: int, d_final_state=None, slopes=None, h_in=None, stream=None):
    """Reversed state entering shard `rank` from its right end: gathered [R, B, H, D, D] holds every shard's
    la_shard_state_reverse in rank order, L the tokens per shard, d_final_state the gradient of the sequences'
    final state (or None). Returns h_in [B, H, D, D] fp32."""
    _need_cuda(gathered, d_final_state, slopes, h_in)
    R, B, H, D, _ = gathered.shape
    if gathered.dtype != torch.float32 or tuple(gathered.shape) != (R, B, H, D, D):
        raise ValueError(f"gathered must be float32 [R, B, H, D, D] (got {tuple(gathered.shape)}, {gathered.dtype})")
    _check_sizes(gathered, states=(("d_final_state", d_final_state, B), ("h_in", h_in, B)), slopes=slopes, H=H, D=D)
    if h_in is None:
        h_in = torch.empty((B, H, D, D), dtype=torch.float32, device=gathered.device)
    st = lib().la_cp_reverse_entry_state(_ptr(gathered), R, rank, B, H, D, L, _ptr(d_final_state), _ptr(slopes),
                                         _ptr(h_in), _stream(stream))
    _check(st, "la_cp_reverse_entry_state")
    return h_in


class CudaShardOps:
    """The per-rank steps of la_prefill_cp and la_prefill_cp_backward, on this GPU through the library."""

    @staticmethod
    def shard_state(k, v, slopes):
        return la_shard_state(k, v, slopes=slopes)

    @staticmethod
    def entry_state(gathered, rank, L, initial_state, slopes):
        return la_cp_entry_state(gathered, rank, L, initial_state=initial_state, slopes=slopes)

    @staticmethod
    def prefill(q, k, v, s_in, return_final_state, slopes, out_dtype):
        return la_prefill(q, k, v, initial_state=s_in, return_final_state=return_final_state, slopes=slopes,
                          out_dtype=out_dtype)

    @staticmethod
    def shard_state_reverse(q, dout, slopes):
        return la_shard_state_reverse(q, dout, slopes=slopes)

    @staticmethod
    def reverse_entry_state(gathered, rank, L, d_final_state, slopes):
        return la_cp_reverse_entry_state(gathered, rank, L, d_final_state=d_final_state, slopes=slopes)

    @staticmethod
    def backward(q, k, v, dout, s_in, h_in, slopes, out_dtype):
        return la_prefill_backward(q, k, v, dout, initial_state=s_in, d_final_state=h_in, return_d_initial_state=True,
                                   slopes=slopes, out_dtype=out_dtype)

    @staticmethod
    def varlen_entry_state(gathered, rank, cu_host, initial_state, slopes):
        return la_cp_varlen_entry_state(gathered, rank, cu_host, initial_state=initial_state, slopes=slopes)

    @staticmethod
    def varlen_reverse_entry_state(gathered, rank, cu_host, d_final_state, slopes):
        return la_cp_varlen_reverse_entry_state(gathered, rank, cu_host, d_final_state=d_final_state, slopes=slopes)

    @staticmethod
    def prefill_varlen(q, k, v, local_cu, init, slopes, out_dtype):
        cu = torch.tensor(local_cu, dtype=torch.int32, device=q.device)
        return la_prefill_varlen(q, k, v, cu, initial_state=init, return_final_state=True, slopes=slopes,
                                 out_dtype=out_dtype)

    @staticmethod
    def backward_varlen(q, k, v, dout, local_cu, init, dfin, slopes, out_dtype):
        cu = torch.tensor(local_cu, dtype=torch.int32, device=q.device)
        return la_prefill_varlen_backward(q, k, v, dout, cu, initial_state=init, d_final_state=dfin,
                                          return_d_initial_state=True, slopes=slopes, out_dtype=out_dtype)


def la_prefill_cp(q, k, v, group=None, initial_state=None, return_final_state=False, slopes=None, out_dtype=None,
                  ops=CudaShardOps):
    """Context-parallel prefill: the sequences of one batch are sharded along N over the ranks of a
    torch.distributed group, rank r holding tokens [r*L, (r+1)*L) of every sequence as q, k, v
    [B, L, H, D]. Each rank computes its shard's state from a zero start, the states are all-gathered
    (the one exchange step), each rank forms the state entering its shard and runs the prefill from it.
    Returns this rank's o (and its final state, which on the last rank is the sequences' final state).
    initial_state, if given, is the sequences' initial state, the same on every rank. `ops` runs the
    per-rank steps (the library's kernels by default)."""
    import torch.distributed as dist
    single = not (dist.is_available() and dist.is_initialized())
    R = 1 if single else dist.get_world_size(group)
    r = 0 if single else dist.get_rank(group)
    L = q.shape[1]
    ds = ops.shard_state(k, v, slopes)
    if single:
        gathered = ds.unsqueeze(0)
    else:
        parts = [torch.empty_like(ds) for _ in range(R)]
        dist.all_gather(parts, ds.contiguous(), group=group)
        gathered = torch.stack(parts)
    s_in = ops.entry_state(gathered, r, L, initial_state, slopes)
    return ops.prefill(q, k, v, s_in, return_final_state, slopes, out_dtype)


def la_prefill_cp_backward(q, k, v, dout, group=None, initial_state=None, d_final_state=None, slopes=None,
                           out_dtype=None, ops=CudaShardOps):
    """Context-parallel backward pass: rank r of a torch.distributed group holds tokens [r*L, (r+1)*L) of
    every sequence (q, k, v and the output gradient dout, [B, L, H, D]); initial_state (the forward's S0)
    and d_final_state (the gradient of the sequences' final state) are the same on every rank, or None.
    Each rank computes its shard's forward state and reversed state from a zero start; both are
    all-gathered in one collective (the one exchange step); each rank forms the forward state entering its
    shard from the left and the reversed state entering it from the right, and runs the backward pass of
    its shard from them. Returns this rank's (dq, dk, dv, d_initial_state): the gradients of its shard,
    and on rank 0 the gradient of the sequences' initial state. `ops` runs the per-rank steps (the
    library's kernels by default)."""
    import torch.distributed as dist
    single = not (dist.is_available() and dist.is_initialized())
    R = 1 if single else dist.get_world_size(group)
    r = 0 if single else dist.get_rank(group)
    L = q.shape[1]
    ds = ops.shard_state(k, v, slopes)
    dh = ops.shard_state_reverse(q, dout, slopes)
    both = torch.stack([ds, dh]).contiguous()
    if single:
        gathered = both.unsqueeze(0)
    else:
        parts = [torch.empty_like(both) for _ in range(R)]
        dist.all_gather(parts, both, group=group)
        gathered = torch.stack(parts)
    s_in = ops.entry_state(gathered[:, 0].contiguous(), r, L, initial_state, slopes)
    h_in = ops.reverse_entry_state(gathered[:, 1].contiguous(), r, L, d_final_state, slopes)
    return ops.backward(q, k, v, dout, s_in, h_in, slopes, out_dtype)


# --------------------------------------------------------------------------- context parallelism over varlen batches
def _host_cu(cu_seqlens):
    """cu_seqlens as a host int32 array (a list, a numpy array or a CPU tensor; not a CUDA tensor: the planning
    is on the host and the caller knows the packing)."""
    import numpy as np
    if isinstance(cu_seqlens, torch.Tensor):
        if cu_seqlens.is_cuda:
            raise ValueError("pass the host copy of cu_seqlens (the packing is planned on the host)")
        cu_seqlens = cu_seqlens.numpy()
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))


def la_cp_varlen_entry_state(gathered, rank: int, cu_seqlens, initial_state=None, slopes=None, s_in=None, stream=None):
    """State entering the first sub-sequence of shard `rank` of a packed batch cut into R equal shards along its
    token axis. gathered [R, H, D, D]: every rank's last-sub-sequence state from a zero start, in rank order;
    cu_seqlens: the host copy of the whole batch's [nseq + 1]; initial_state [nseq, H, D, D] or None.
    Returns s_in [H, D, D] fp32."""
    _need_cuda(gathered, initial_state, slopes, s_in)
    R, H, D, _ = gathered.shape
    cu = _host_cu(cu_seqlens)
    nseq = cu.size - 1
    if gathered.dtype != torch.float32 or tuple(gathered.shape) != (R, H, D, D):
        raise ValueError(f"gathered must be float32 [R, H, D, D] (got {tuple(gathered.shape)}, {gathered.dtype})")
    _check_sizes(gathered, states=(("initial_state", initial_state, nseq),), slopes=slopes, H=H, D=D)
    if s_in is None:
        s_in = torch.empty((H, D, D), dtype=torch.float32, device=gathered.device)
    elif tuple(s_in.shape) != (H, D, D) or s_in.dtype != torch.float32:
        raise ValueError("s_in must be float32 [H, D, D]")
    st = lib().la_cp_varlen_entry_state(_ptr(gathered), R, rank, ctypes.c_void_p(cu.ctypes.data), nseq, H, D,
                                        _ptr(initial_state), _ptr(slopes), _ptr(s_in), _stream(stream))
    _check(st, "la_cp_varlen_entry_state")
    return s_in


def la_cp_varlen_reverse_entry_state(gathered, rank: int, cu_seqlens, d_final_state=None, slopes=None, h_in=None,
                                     stream=None):
    """Reversed state entering the last sub-sequence of shard `rank` from its right end. gathered [R, H, D, D]:
    every rank's first-sub-sequence reversed state from a zero start; d_final_state [nseq, H, D, D] or None.
    Returns h_in [H, D, D] fp32."""
    _need_cuda(gathered, d_final_state, slopes, h_in)
    R, H, D, _ = gathered.shape
    cu = _host_cu(cu_seqlens)
    nseq = cu.size - 1
    if gathered.dtype != torch.float32 or tuple(gathered.shape) != (R, H, D, D):
        raise ValueError(f"gathered must be float32 [R, H, D, D] (got {tuple(gathered.shape)}, {gathered.dtype})")
    _check_sizes(gathered, states=(("d_final_state", d_final_state, nseq),), slopes=slopes, H=H, D=D)
    if h_in is None:
        h_in = torch.empty((H, D, D), dtype=torch.float32, device=gathered.device)
    elif tuple(h_in.shape) != (H, D, D) or h_in.dtype != torch.float32:
        raise ValueError("h_in must be float32 [H, D, D]")
    st = lib().la_cp_varlen_reverse_entry_state(_ptr(gathered), R, rank, ctypes.c_void_p(cu.ctypes.data), nseq, H, D,
                                                _ptr(d_final_state), _ptr(slopes), _ptr(h_in), _stream(stream))
    _check(st, "la_cp_varlen_reverse_entry_state")
    return h_in


class VarlenShard:
    """The sub-sequences of shard `rank` when a packed batch (cu_seqlens over T tokens) is cut into R equal shards
    [rank L, (rank+1) L), L = T / R: the sequences meeting the shard, in order, each clipped to it; an empty
    sequence at token p belongs to the rank holding token p (the last rank for p = T).
      subs            [(sequence, a, b)] global token range [a, b) of each sub-sequence
      local_cu        cu_seqlens of the sub-sequences within the shard (int list, starting at 0)
      starts_here     per sub-sequence: it is its sequence's beginning (it takes its initial state)
      ends_here       per sub-sequence: it is its sequence's end (its final state is the sequence's)
      first_continues the first sub-sequence began on an earlier rank
      last_continues  the last sub-sequence goes on on a later rank"""

    def __init__(self, cu_seqlens, R: int, rank: int):
        cu = [int(x) for x in _host_cu(cu_seqlens)]
        nseq = len(cu) - 1
        T = cu[-1]
        if nseq < 1 or T <= 0 or T % R or not 0 <= rank < R:
            raise ValueError(f"need nseq >= 1, T = {T} > 0 divisible by R = {R}, and 0 <= rank < R")
        if cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])):
            raise ValueError("cu_seqlens must start at 0 and be non-decreasing")
        L = T // R
        s, e = rank * L, (rank + 1) * L
        self.R, self.rank, self.L, self.s, self.e, self.cu = R, rank, L, s, e, cu
        self.subs = []
        for i in range(nseq):
            a, b = cu[i], cu[i + 1]
            if a == b:
                if min(a // L, R - 1) == rank:
                    self.subs.append((i, a, a))
            elif a < e and b > s:
                self.subs.append((i, max(a, s), min(b, e)))
        self.local_cu = [0]
        for _, a, b in self.subs:
            self.local_cu.append(self.local_cu[-1] + b - a)
        self.seqs = [i for i, _, _ in self.subs]
        self.starts_here = [cu[i] >= s for i in self.seqs]
        self.ends_here = [cu[i + 1] <= e for i in self.seqs]
        self.first_continues = not self.starts_here[0]
        self.last_continues = not self.ends_here[-1]


def _gather(x, group):
    """[R, *x.shape]: every rank's x in rank order (x itself when no process group is initialised)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return x.unsqueeze(0)
    parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def _rank_world(group):
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 0, 1
    return dist.get_rank(group), dist.get_world_size(group)


def varlen_cp_send(k, v, shard: "VarlenShard", slopes=None, ops=None, q=None, dout=None):
    """This rank's part of the all-gather: the state its last sub-sequence produces from a zero start ([H, D, D]);
    with q and dout (the backward pass) also the reversed state its first sub-sequence produces from a zero
    start, stacked: [2, H, D, D]."""
    ops = CudaShardOps if ops is None else ops
    a = shard.local_cu[-2]
    fwd = ops.shard_state(k[a:].unsqueeze(0), v[a:].unsqueeze(0), slopes)[0]
    if q is None:
        return fwd
    b = shard.local_cu[1]
    rev = ops.shard_state_reverse(q[:b].unsqueeze(0), dout[:b].unsqueeze(0), slopes)[0]
    return torch.stack([fwd, rev])


def _sub_states(shard, first, given, like):
    """[n, H, D, D]: `first` for the first sub-sequence, the given per-sequence states (or zeros) for the others."""
    out = torch.zeros((len(shard.subs),) + tuple(first.shape), dtype=first.dtype, device=like.device)
    out[0] = first
    if given is not None:
        for j, i in enumerate(shard.seqs[1:], start=1):
            out[j] = given[i]
    return out


def varlen_cp_forward(q, k, v, shard: "VarlenShard", gathered, initial_state=None, return_final_state=False,
                      slopes=None, out_dtype=None, ops=None):
    """This rank's outputs from the gathered states: the entry state of its first sub-sequence, then one varlen
    prefill over its sub-sequences. Returns o, or (o, final_states, seq_ids) with the final states of the
    sequences that end on this rank."""
    ops = CudaShardOps if ops is None else ops
    s_in = ops.varlen_entry_state(gathered, shard.rank, shard.cu, initial_state, slopes)
    init = _sub_states(shard, s_in, initial_state, q)
    o, fin = ops.prefill_varlen(q, k, v, shard.local_cu, init, slopes, out_dtype)
    if not return_final_state:
        return o
    ends = [j for j, x in enumerate(shard.ends_here) if x]
    return o, fin[ends], [shard.seqs[j] for j in ends]


def varlen_cp_backward(q, k, v, dout, shard: "VarlenShard", gathered, initial_state=None, d_final_state=None,
                       slopes=None, out_dtype=None, ops=None):
    """This rank's gradients from the gathered states ([R, 2, H, D, D]: forward and reversed): the entry state of
    its first sub-sequence and the reversed entry state of its last, then one varlen backward pass over its
    sub-sequences. Returns (dq, dk, dv, d_initial_states, seq_ids) with the initial-state gradients of the
    sequences that start on this rank."""
    ops = CudaShardOps if ops is None else ops
    s_in = ops.varlen_entry_state(gathered[:, 0].contiguous(), shard.rank, shard.cu, initial_state, slopes)
    h_in = ops.varlen_reverse_entry_state(gathered[:, 1].contiguous(), shard.rank, shard.cu, d_final_state, slopes)
    init = _sub_states(shard, s_in, initial_state, q)
    dfin = torch.zeros_like(init)
    if d_final_state is not None:
        for j, i in enumerate(shard.seqs[:-1]):
            dfin[j] = d_final_state[i]
    dfin[-1] = h_in
    dq, dk, dv, dinit = ops.backward_varlen(q, k, v, dout, shard.local_cu, init, dfin, slopes, out_dtype)
    starts = [j for j, x in enumerate(shard.starts_here) if x]
    return dq, dk, dv, dinit[starts], [shard.seqs[j] for j in starts]


def la_prefill_varlen_cp(q, k, v, cu_seqlens, group=None, initial_state=None, return_final_state=False, slopes=None,
                         out_dtype=None, ops=None):
    """Context-parallel varlen prefill: a packed batch (host cu_seqlens over T tokens) is cut along its token
    axis into R equal shards over the ranks of a torch.distributed group; this rank holds tokens
    [rank L, (rank+1) L) as q, k, v [L, H, D]. Each rank computes the state of its last sub-sequence from a
    zero start, the states are all-gathered (the one exchange step), and each rank forms the state entering its
    first sub-sequence and runs one varlen prefill over its sub-sequences. Returns this rank's o, or
    (o, final_states, seq_ids): the final states of the sequences that end on this rank and their indices.
    initial_state [nseq, H, D, D] (the same on every rank) or None. `ops` runs the per-rank steps (the library's
    kernels by default)."""
    rank, world = _rank_world(group)
    shard = VarlenShard(cu_seqlens, world, rank)
    gathered = _gather(varlen_cp_send(k, v, shard, slopes, ops), group)
    return varlen_cp_forward(q, k, v, shard, gathered, initial_state, return_final_state, slopes, out_dtype, ops)


def la_prefill_varlen_cp_backward(q, k, v, dout, cu_seqlens, group=None, initial_state=None, d_final_state=None,
                                  slopes=None, out_dtype=None, ops=None):
    """Context-parallel varlen backward pass over the shards of la_prefill_varlen_cp (dout [L, H, D] this rank's
    output gradients; initial_state and d_final_state [nseq, H, D, D] or None, the same on every rank). Each
    rank computes its last sub-sequence's state and its first sub-sequence's reversed state from a zero start;
    both travel in one all-gather; each rank forms both entry states and runs one varlen backward pass.
    Returns (dq, dk, dv, d_initial_states, seq_ids): this rank's gradients and the initial-state gradients of
    the sequences that start on it."""
    rank, world = _rank_world(group)
    shard = VarlenShard(cu_seqlens, world, rank)
    gathered = _gather(varlen_cp_send(k, v, shard, slopes, ops, q=q, dout=dout), group)
    return varlen_cp_backward(q, k, v, dout, shard, gathered, initial_state, d_final_state, slopes, out_dtype, ops)
