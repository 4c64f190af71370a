"""Float64 CPU oracle for exact masked attention.

TEST INFRASTRUCTURE ONLY: only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import it.  It shares no code with the CUDA
library.  See oracle/definition.py for the definition and its citations.
"""
from .definition import (alibi_bias, alibi_slopes, attention, attention_bh, attention_head,
                         attention_weights, keep_mask, kept_pairs, kv_head_of, scores)
from .backward import attention_backward, backward_head, row_dot, tiled_backward_head
from .decode import decode, decode_split, merge_partials, partial_head, positions
from .tiled import tiled_attention, tiled_kv_outer, tiled_q_outer

__all__ = [
    "alibi_bias", "alibi_slopes", "attention", "attention_backward", "attention_bh",
    "attention_head", "backward_head", "decode", "row_dot", "tiled_backward_head",
    "decode_split", "merge_partials", "partial_head", "positions",
    "attention_weights", "keep_mask", "kept_pairs", "kv_head_of", "scores", "tiled_attention",
    "tiled_kv_outer", "tiled_q_outer",
]
