"""Exact IO-aware scaled-dot-product attention for B200 (sm_100a).

The public API is the C-ABI library ``libattn.so`` (``include/attn.h``) and its
Python binding :mod:`exact_io_aware_57_b200.attn`; the names below are loaded
from the binding on first use so that the build script and the input
generators import without the compiled library.
"""
_BINDING_NAMES = {
    "attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_fwd_varlen", "attn_fwd_naive",
    "attn_naive_scratch_size", "attn_device_status", "attn_launch_count", "AttnError",
    "attn_fwd_splitkv", "attn_splitkv_num_splits", "attn_splitkv_workspace_size", "attn_merge_partials", "attn_bwd_varlen", "attn_fwd_dv",
    "attn_fwd_partial", "attn_bwd_dv", "attn_quantize_e4m3", "attn_fwd_fp8",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import attn as _attn

        return getattr(_attn, name)
    raise AttributeError(name)
