"""Seeded synthetic workloads for the expert-balance path.

This package only draws inputs: gate top-k expert ids shaped like the routing
of the MoE models named on the UltraEP page ("300 µs to level MoE expert load",
section "How UltraEP balances in real time within 300 µs") and the Waterfill
page (section "Experimental setup"), plus bf16 tensors for hidden states,
expert weights and replica gradients.  It holds none of the balancing
arithmetic, so both the CUDA path and the CPU oracle may consume it.
"""
from .configs import CONFIGS, WorkloadConfig, get_config
from .routing import topk_ids, hidden_states_np, expert_weights_np, replica_grads_np

__all__ = [
    "CONFIGS",
    "WorkloadConfig",
    "get_config",
    "topk_ids",
    "hidden_states_np",
    "expert_weights_np",
    "replica_grads_np",
]
