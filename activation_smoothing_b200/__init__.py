"""Rotated Runtime Smooth (RRS) W4A4 linear layer for NVIDIA B200 (sm_100a).

The computation runs in the CUDA library ``librrs.so`` (C ABI in
``include/rrs.h``); this package is its thin Python binding plus the seeded
synthetic workloads.  Build the library with
``python -m activation_smoothing_b200.build``.
"""
from . import workloads  # noqa: F401  (no CUDA needed)

_API = (
    "NO_ROTATE", "FORCE_UNIT_SCALES", "WS_HOLDS_A8", "W_EXPANDED", "Y_BF16", "Y_SILU_MUL", "ONE_LAUNCH", "interleave_gate_up", "RRSError", "lib", "workspace_size", "make_workspace",
    "prepare_weights", "smooth_quant", "group_max", "smooth_quant_scaled", "w4a4_gemm", "linear", "linear_from_host",
    "w4a4_gemm_debug_partials", "channel_absmax", "perm_from_channel_max", "calibrate_perm",
    "check_workspace", "check_perm", "debug_wait_timeout", "debug_divide", "expand_weights", "silu_mul", "kv_quant", "kv_dequant", "LIB_PATH",
)


def __getattr__(name):
    # The binding is imported on first use so that the workloads module can be
    # used on machines where the library has not been built.
    if name in _API:
        from . import _binding
        return getattr(_binding, name)
    raise AttributeError(name)


__all__ = list(_API) + ["workloads"]
