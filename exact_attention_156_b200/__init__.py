"""B200 (sm_100a) exact attention: fused forward with online softmax and a
recompute-based backward, behind the C ABI of include/attn.h.

    from exact_attention_156_b200 import attn_fwd, attn_bwd
    o, lse = attn_fwd(q, k, v, causal=True)              # q, k, v: bf16 (B, S, H, D) CUDA
    dq, dk, dv = attn_bwd(q, k, v, o, do, lse, causal=True)
    o, lse = attn_decode(q_new, k_cache, v_cache, cache_seqlens, causal=True)  # KV-cache decode
    o, lse = attn_fwd_varlen(q, k, v, cu_q, cu_k, max_q, max_k, causal=True)   # packed batches
    o, lse = attn_fwd_padded(q, k, v, seqlens_q, seqlens_k, causal=True)       # padded batches
"""
from ._binding import (  # noqa: F401
    ATTN_STATUS,
    LIB_PATH,
    AttnError,
    attn_bwd,
    attn_bwd_padded,
    attn_bwd_padded_workspace_size,
    attn_bwd_stages,
    attn_bwd_varlen,
    attn_bwd_varlen_workspace_size,
    attn_bwd_workspace_size,
    attn_decode,
    attn_decode_workspace_size,
    attn_fwd,
    attn_fwd_padded,
    attn_fwd_padded_workspace_size,
    attn_fwd_varlen,
    decode_split_plan,
    device_timeout_selftest,
    get_last_device_error,
    lib,
    status_string,
)
