"""fp64 CPU oracle for causal self-attention: TEST INFRASTRUCTURE.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this package.  The product library never does, and this package
imports nothing from the product.
"""

from .attention import (attention_backward, attention_backward_given_o,
                        attention_backward_heads, attention_forward,
                        attention_forward_heads, attention_rows, causal_mask,
                        delta_from_o, head_probs)

__all__ = [
    "attention_forward", "attention_backward", "attention_forward_heads",
    "attention_backward_heads", "attention_backward_given_o", "attention_rows", "causal_mask",
    "delta_from_o", "head_probs",
]
