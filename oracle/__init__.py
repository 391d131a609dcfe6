"""fp64 CPU oracle of the routed MoE FFN layer -- test infrastructure only.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg may
import it; the product path never does. See ``moe_oracle`` for what it computes.
"""
from .moe_oracle import (E4M3_MAX, Fp8Experts, bf16_to_f64, combine,  # noqa: F401
                         compact_zero_channels, dequantize_fp8_rows, e4m3_decode, e4m3_encode,
                         expert_outputs_packed, forward_inputs, live_channels, moe_forward,
                         permute, quantize_fp8_rows, router_logits, routing_weights,
                         shared_gate, sigmoid, silu, swiglu_expert, topk_select)
