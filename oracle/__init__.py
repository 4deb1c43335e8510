"""CPU fp64 oracle of the top-k MoE FFN layer forward (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package.  The CUDA library never uses it.
"""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (  # noqa: F401
    LayerResult, PlanInfeasible, PlanStats, Segments, balanced_plan, capacity_rows, combine,
    dispatch_positions, enforce_margin, expert_ffn, expert_rank, f64, grouped_expert_ffn,
    histogram, i64, layer_forward, margin_violations, num_segments, permute_rows,
    plain_segments, route, router_logits, shared_expert, silu, token_output, topk_ids, topk_weights,
    topk_weights_softmax_all, ExpertChoice, expert_choice, expert_choice_forward, expert_scores,
    select_tokens, ec_margin_violations, enforce_ec_margin, combine_expert_choice, expert_choice_map,
    Rerouted, candidate_order, reroute_overflow, reroute_positions, layer_forward_reroute,
)
