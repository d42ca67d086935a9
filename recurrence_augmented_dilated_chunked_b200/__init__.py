"""B200-native (sm_100a) RAT+ sequence mixer.

The hot path of RAT+ (recurrence-augmented dilated attention): the
full-sequence forget-gate recurrence over the key and value streams, dilated
(+ windowed, + head-wise hybrid) causal attention over the recurrent keys and
values, and the fused decode step over a D-compressed KV cache.  All compute
runs in hand-written CUDA kernels behind the C ABI of ``include/ratp.h``; this
package is the thin ctypes binding plus the seeded input generators.
"""
from ._binding import (  # noqa: F401
    KVCache,
    RatpError,
    attn_workspace,
    dilated_attn_prefill,
    dilated_attn_prefill_per_sample,
    dilated_attn_prefill_simt,
    debug_fault,
    decode_step_layers,
    exported_symbols,
    guard_line,
    last_error,
    load_library,
    prefill_fused,
    prefill_fused_workspace,
    scan_prefill,
    scan_prefill_kv,
    scan_prefill_kv_noalloc,
    scan_prefill_kv_window,
    scan_workspace,
    sm_count,
)
from .inputs import WORKLOADS, Workload, decode_context, decode_inputs, prefill_inputs  # noqa: F401
