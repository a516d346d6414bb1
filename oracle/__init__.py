"""CPU oracle for the sparse noisy top-k MoE layer forward pass.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg use it; the product path never does.
"""
from .oracle import (  # noqa: F401
    build, capacity, router_logits, route_from_logits, assign_slots, load_stats, backward, backward_sampled,
    expert_ffn,
    expert_ffn_ex, ffn_combine, forward, ORACLE_F32, ORACLE_BF16, ACT_RELU, ACT_GELU,
)
