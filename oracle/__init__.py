"""Float64 CPU oracle for causal self-attention (test infrastructure only; never on the product path)."""
from .attn_ref import (attention_backward, attention_forward, causal_flops, causal_mask, head_backward,
                       head_forward, slice_forward_backward)

__all__ = ["attention_forward", "attention_backward", "head_forward", "head_backward", "causal_mask",
           "slice_forward_backward", "causal_flops"]
