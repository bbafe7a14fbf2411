"""fp64 CPU oracle for exact attention -- test infrastructure, never part of the product path."""
from .attention import (attention_forward, attention_forward_online, attention_backward,
                        attention_probs, attention_rows, attention_dq_rows, attention_row_stats,
                        attention_dkdv_key_rows, attention_forward_gqa, attention_backward_gqa,
                        attention_forward_rect)

__all__ = ["attention_forward", "attention_forward_online", "attention_backward",
           "attention_probs", "attention_rows", "attention_dq_rows", "attention_row_stats",
           "attention_dkdv_key_rows", "attention_forward_gqa", "attention_backward_gqa",
           "attention_forward_rect"]
