"""fp64 CPU oracle for the Dual-Flow decode step.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA library.
"""

from .dualflow_oracle import (  # noqa: F401
    bf16_round,
    couple_query,
    gather_kv,
    attn_weights,
    decode_attn,
    kv_append,
    prefill,
    grouped_proj,
    silu,
    swiglu_couple,
    residual_couple,
    rmsnorm,
    layer_step,
    LAYER_INTERFACES,
    softmax_rows,
    collision_probability,
    mixture_weight,
    mixture_head,
    moe_route,
    moe_expert,
    moe_forward,
)
