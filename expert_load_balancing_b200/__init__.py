"""B200-native sigmoid MoE router with Exact Quantile Balancing (EQB).

The routing path, and the expert layer after it (dispatch, grouped SwiGLU
projections, combine), run in ``libkolibri_router.so`` (hand-written sm_100a CUDA
behind the C ABI in ``include/kolibri_router.h``).  ``binding`` is the thin
ctypes layer with the same call names; ``workloads`` draws seeded synthetic
inputs; ``build`` compiles the library in-tree.
"""
from . import binding  # noqa: F401  (loads the library lazily, on first call)
from .binding import (  # noqa: F401
    KolibriError,
    expert_ffn_workspace,
    kolibri_device_status,
    kolibri_eqb_bf16_bias,
    kolibri_eqb_bf16_digit,
    kolibri_eqb_bf16_histogram,
    kolibri_eqb_key_bias,
    kolibri_eqb_key_digit,
    kolibri_eqb_key_histogram,
    kolibri_eqb_update,
    kolibri_eqb_update_bf16,
    kolibri_expert_combine,
    kolibri_expert_dispatch,
    kolibri_expert_down,
    kolibri_expert_ffn,
    kolibri_expert_gate_up,
    kolibri_expert_permute,
    kolibri_expert_permute_noalloc,
    kolibri_intervention_rate,
    kolibri_lei_inject,
    kolibri_route_and_balance,
    kolibri_router_forward,
    kolibri_router_forward_eqb,
    kolibri_router_forward_permute,
    kolibri_router_logits,
    kolibri_router_topk,
    kolibri_score_grad_to_logits,
    kolibri_selftest_bounded_wait,
    kolibri_workspace_bytes,
    workspace,
)
