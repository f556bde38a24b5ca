"""Local MoE expert forward on the non-expand routed layout, for NVIDIA B200 (sm_100a).

The computation lives in ``libmoe_nonexpand.so`` (C ABI: include/moe_nonexpand.h);
``binding`` passes torch tensors' device pointers and the current stream to it.
"""
from .binding import (  # noqa: F401
    ACT_SWIGLU, LAYOUT_CONCATENATED, LAYOUT_INTERLEAVED, MoeError, alloc_meta,
    alloc_workspace, combine, forward, intermediates_from_workspace, meta_from_workspace,
    metadata, read_error, workspace_bytes, workspace_layout,
)
