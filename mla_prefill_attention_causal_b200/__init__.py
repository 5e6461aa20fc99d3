"""MLA prefill attention for NVIDIA B200 (sm_100a).

The computation lives in ``libmla.so`` (hand-written CUDA, C ABI declared in
``include/mla.h``); this package is its thin Python binding.  PyTorch only
provides device memory and the current stream.
"""
from ._lib import (  # noqa: F401
    LIB_PATH,
    MlaError,
    load,
    mla_attn_merge,
    mla_debug_wait_timeout,
    mla_device_status,
    mla_prefill_fwd,
    mla_prefill_fwd_context,
    mla_prefill_fwd_dims,
    mla_prefill_fwd_ex,
    mla_prefill_fwd_splitkv,
    num_splits_for,
    mla_sparse_prefill_fwd,
    prefill_workspace_size,
    splitkv_workspace_size,
    status_string,
)
