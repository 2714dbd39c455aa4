"""B200-native (sm_100a) Lightning Attention: chunked prefill, varlen prefill, their backward pass, decode.

The operator and its C ABI are described in include/la.h; ``binding`` exposes
the same entry points on torch tensors. The CUDA library is loaded lazily, on
the first call, so that importing the package (for instance for the seeded
input generators in ``inputs``) needs no GPU.
"""

from .binding import (  # noqa: F401
    EXPORTS,
    LAError,
    la_cp_entry_state,
    la_cp_reverse_entry_state,
    la_cp_varlen_entry_state,
    la_cp_varlen_reverse_entry_state,
    la_decode_step,
    la_decode_steps,
    la_decode_steps_norm_gate,
    la_get_device_error,
    la_last_error,
    la_last_launch_count,
    la_norm_gate,
    la_prefill,
    la_prefill_backward,
    la_prefill_backward_workspace_size,
    la_prefill_cp,
    la_prefill_cp_backward,
    la_prefill_noalloc,
    la_prefill_norm_gate,
    la_prefill_varlen,
    la_prefill_varlen_backward,
    la_prefill_varlen_backward_workspace_size,
    la_prefill_varlen_cp,
    la_prefill_varlen_cp_backward,
    la_prefill_varlen_norm_gate,
    la_prefill_varlen_workspace_size,
    la_prefill_workspace_size,
    la_shard_state,
    la_shard_state_reverse,
    la_shard_state_workspace_size,
    la_status_string,
    la_trace_collect,
    la_trace_enable,
    la_validate_cu_seqlens,
)
