"""HSTU pointwise jagged attention on NVIDIA B200 (sm_100a).

The work runs in libhstu.so (hand-written CUDA: tcgen05/TMEM/TMA attention,
LayerNorm-gate epilogue, paged-KV gather, exact time buckets; the layer's
f1/f2 projections on cuBLASLt with an in-place SiLU kernel; the paged KV
cache's append/evict kernels), reached
through its C ABI (include/hstu.h).  This package is the thin Python binding.
"""
from ._lib import AttnParams, HstuError, LIB_PATH  # noqa: F401
from .api import (  # noqa: F401
    attn_params,
    hstu_attn_bwd,
    hstu_attn_fwd,
    hstu_attn_fwd_paged,
    hstu_attn_paged_default_splits,
    hstu_attn_paged_workspace_size,
    hstu_attn_workspace_size,
    hstu_check_device_error,
    hstu_status_string,
    hstu_kv_append,
    hstu_kv_evict,
    hstu_kv_workspace_size,
    hstu_layer_f1,
    hstu_layer_f2,
    hstu_linear,
    hstu_linear_workspace_size,
    hstu_mfalcon_fwd,
    hstu_mfalcon_workspace_size,
    hstu_ts_bucket,
    hstu_version,
    split_uvqk,
)

__all__ = [
    "AttnParams", "HstuError", "attn_params", "hstu_attn_fwd", "hstu_attn_fwd_paged",
    "hstu_attn_paged_default_splits", "hstu_attn_paged_workspace_size", "hstu_attn_workspace_size",
    "hstu_check_device_error", "hstu_status_string", "hstu_ts_bucket", "hstu_version",
    "hstu_layer_f1", "hstu_layer_f2", "hstu_linear", "hstu_linear_workspace_size", "split_uvqk",
    "hstu_kv_append", "hstu_kv_evict", "hstu_kv_workspace_size", "hstu_mfalcon_fwd",
    "hstu_mfalcon_workspace_size", "hstu_attn_bwd",
]
