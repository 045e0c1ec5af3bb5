"""CPU fp64 oracle of the MoE layer (test infrastructure; see moe_oracle.py)."""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (P_PAD, forward, backward, router_logits, topk_ids, gates,  # noqa: F401
                         schedule, silu, silu_grad, token_forward_backward,
                         mx_quantize, mx_dequantize, e4m3_encode, e4m3_decode)
