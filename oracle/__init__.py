"""fp64 CPU oracle of the routed MoE FFN layer -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it; the product path never does. See ``moe_oracle`` for what it computes.
"""
from .moe_oracle import (bf16_to_f64, combine, compact_zero_channels,  # noqa: F401
                         expert_outputs_packed, forward_inputs, live_channels, moe_forward,
                         permute, router_logits, routing_weights, shared_gate, sigmoid, silu,
                         swiglu_expert, topk_select)
