"""Dual-Flow Transformer decode step on NVIDIA B200 (sm_100a).

The compute lives in libdualflow.so (C ABI, include/dualflow.h); this
package is its thin binding plus the layer-step composition.
"""

from .api import (  # noqa: F401
    decode_attn,
    decode_attn_num_launches,
    decode_attn_num_splits,
    decode_attn_workspace_size,
    grouped_proj,
    grouped_proj_batched,
    grouped_proj_num_launches,
    grouped_proj_workspace_size,
    kv_append,
    mixture_head,
    mixture_head_slices,
    moe_combine,
    moe_dispatch,
    moe_route,
    new_attn_workspace,
    new_prefill_workspace,
    new_proj_workspace,
    prefill,
    prefill_num_launches,
    prefill_workspace_size,
    rmsnorm,
)
