"""Oracle package: the float64 CPU restatement of the DeepSeekMoE layer forward.

Test infrastructure only; see dsmoe_oracle.py.
"""
from .dsmoe_oracle import *  # noqa: F401,F403
from .dsmoe_oracle import (bf16_bits_to_f64, router_logits, scores, select_topk, hash_route,
                           balance_stats, swiglu_ffn, swiglu_hidden, moe_layer, route, forward, combinations,
                           sigmoid, softplus, sqrt_softplus, softmax, silu)
