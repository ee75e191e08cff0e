"""Float64 CPU oracle for causal self-attention (test infrastructure only; never on the product path)."""
from .attn_ref import (attention_backward, attention_forward, causal_mask, decode_forward, head_backward,
                       head_forward, kv_group, qk_norm_rope, qk_norm_rope_backward, slice_forward_backward)

__all__ = ["attention_forward", "attention_backward", "head_forward", "head_backward", "causal_mask", "kv_group",
           "slice_forward_backward", "decode_forward", "qk_norm_rope", "qk_norm_rope_backward"]
