"""CPU oracle for exact attention (test infrastructure only).

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg may import this package.  The CUDA path never calls it and shares no
code with it.
"""
from .attn_ref import (  # noqa: F401
    attention_backward,
    attention_backward_head,
    attention_backward_kv_head,
    attention_backward_rows,
    attention_backward_rows_dq,
    attention_backward_varlen,
    attention_decode,
    attention_forward,
    attention_forward_rows,
    attention_forward_varlen,
    kv_head,
    online_softmax_forward,
    visible_mask,
)
