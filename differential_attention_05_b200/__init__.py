"""B200-native differential attention (DIFF Transformer V1 / V2 operator).

The compute path is the C-ABI library libdiffattn.so (hand-written sm_100a kernels,
declared in include/diffattn.h). This package is a thin ctypes binding over it; the
functions load the library on first use and raise if it is missing.

Entry points (same names as the C functions):
  diffattn_lambda               lambda and lambda_init on the device
  diffattn_fwd_prefill          fused prefill, V1 / V2, bf16 (tensor cores) or fp32; causal,
                                full, chunked (k, v longer than q) and sliding window
  diffattn_fwd_prefill_varlen   the same over sequences packed back to back (cu_seqlens)
  diffattn_fwd_decode           V2 split-KV decode (and diffattn_fwd_decode_static)
  diffattn_fwd_decode_v1        V1 split-KV decode with the per-head norm
  diffattn_fwd_decode_paged     either decode over a paged cache (block table)
  diffattn_bwd_prefill          gradients dq, dk, dv, dlambda of the prefill
  diffattn_lambda_bwd           gradients of the four lambda vectors
"""
from ._binding import (  # noqa: F401
    DiffattnError,
    diffattn_lambda,
    diffattn_fwd_prefill,
    diffattn_fwd_prefill_varlen,
    diffattn_bwd_prefill,
    diffattn_bwd_workspace_size,
    diffattn_lambda_bwd,
    diffattn_fwd_prefill_train,
    diffattn_bwd_prefill_saved,
    diffattn_fwd_decode,
    diffattn_fwd_decode_static,
    diffattn_fwd_decode_v1,
    diffattn_fwd_decode_paged,
    diffattn_selftest_timeout,
    diffattn_selftest_exp2,
    diffattn_debug_bounds_violations,
    diffattn_decode_workspace_size,
    diffattn_status_string,
    library_path,
    load_library,
)

__all__ = [
    "DiffattnError",
    "diffattn_lambda",
    "diffattn_fwd_prefill",
    "diffattn_fwd_prefill_varlen",
    "diffattn_bwd_prefill",
    "diffattn_bwd_workspace_size",
    "diffattn_lambda_bwd",
    "diffattn_fwd_prefill_train",
    "diffattn_bwd_prefill_saved",
    "diffattn_fwd_decode",
    "diffattn_fwd_decode_static",
    "diffattn_fwd_decode_v1",
    "diffattn_fwd_decode_paged",
    "diffattn_selftest_timeout",
    "diffattn_selftest_exp2",
    "diffattn_debug_bounds_violations",
    "diffattn_decode_workspace_size",
    "diffattn_status_string",
    "library_path",
    "load_library",
]
