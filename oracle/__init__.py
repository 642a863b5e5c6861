"""CPU float64 oracle for the exact attention forward, its gradients and its block.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The CUDA path never imports it.
"""
from .attention import (  # noqa: F401
    apply_causal_mask, attention_f64, attention_head_rows, attention_probs_f64,
    brute_force, logsumexp_rows, online_softmax_f64, scores, softmax_rows,
    to_f64, weighted_sum,
)
from .backward import (  # noqa: F401
    attention_backward_f64, grad_k, grad_p, grad_q, grad_scores, grad_v, recompute_probs,
    row_dot,
)
from .block import attention_block_f64, linear, merge_heads, split_qkv  # noqa: F401
from .fp8 import attention_fp8_f64, decode_e4m3, dequantize_e4m3, untranspose_v  # noqa: F401
