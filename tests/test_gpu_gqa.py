"""Grouped K/V heads (GQA; MQA with one K/V head): forward and backward of the
CUDA path against the float64 oracle on the same seeded inputs, with the
parity bars of the other GPU tests.  dK and dV of a shared K/V head are the
sums over its query heads."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grad, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # B, Sq, Sk, H, Hk, D, causal, wl, wr
    (2, 384, 384, 8, 2, 128, 1, -1, -1),
    (1, 300, 300, 4, 1, 64, 0, -1, -1),      # multi-query, ragged
    (1, 200, 456, 4, 2, 128, 1, -1, -1),     # Sq < Sk, bottom-right causal
    (1, 512, 512, 6, 3, 128, 1, 130, 0),     # sliding window
    (2, 257, 257, 4, 4, 64, 1, -1, -1),      # Hk = H: the ungrouped path
]


def _run(bits, causal, wl, wr, scale, stages=False):
    import torch
    from exact_attention_156_b200 import (attn_bwd, attn_bwd_stages, attn_bwd_workspace_size,
                                          attn_fwd, get_last_device_error)
    q, k, v, do = (to_device(bits[n]) for n in ("q", "k", "v", "do"))
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=(wl, wr))
    if stages:
        B, Sq, H, D = q.shape
        ws = torch.empty(attn_bwd_workspace_size(B, Sq, H, D), dtype=torch.uint8, device="cuda")
        dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
        attn_bwd_stages(q, k, v, o, do, lse, dq, dk, dv, ws, softmax_scale=scale,
                        causal=bool(causal), window_size=(wl, wr))
    else:
        dq, dk, dv = attn_bwd(q, k, v, o, do, lse, softmax_scale=scale, causal=bool(causal),
                              window_size=(wl, wr))
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    return o, lse, dq, dk, dv


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_grouped_heads_forward_and_backward(case):
    B, Sq, Sk, H, Hk, D, causal, wl, wr = case
    bits = make_inputs(B, Sq, Sk, H, D, 3000 + sum(case), 1.0, with_dout=True, Hk=Hk)
    scale = 1.0 / np.sqrt(D)
    o, lse, dq, dk, dv = _run(bits, causal, wl, wr, scale, stages=(case[0] == 2))
    assert tuple(dk.shape) == (B, Sk, Hk, D) and tuple(dv.shape) == (B, Sk, Hk, D)
    ref = oracle.attention_backward(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                    f64(bits["do"]), scale, causal, wl, wr)
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), ref["o"], ref["lse"], str(case))
    floor = 1e-3 * max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(to_f64(g), ref[name], f"{case} {name}", floor)


def test_grouped_heads_h32_hk8_s4096_sampled():
    """B1 H32 Hk8 S4096 D128 causal (x0.5 inputs): O and LSE on sampled rows of
    every query head; dQ on the same rows; dK and dV of two K/V heads in full
    (each the sum over its four query heads)."""
    B, S, H, Hk, D = 1, 4096, 32, 8, 128
    bits = make_inputs(B, S, S, H, D, 3100, 0.5, with_dout=True, Hk=Hk)
    scale = 1.0 / np.sqrt(D)
    o, lse, dq, dk, dv = _run(bits, 1, -1, -1, scale)
    rng = np.random.default_rng(17)
    trip = np.array([(0, h, i) for h in range(H) for i in
                     sorted(set(rng.choice(S, 48, replace=False).tolist()) | {0, S - 1})])
    q64, k64, v64, do64 = (f64(bits[n]) for n in ("q", "k", "v", "do"))
    o_r, lse_r = oracle.attention_forward_rows(q64, k64, v64, trip, scale, 1)
    o_g = to_f64(o)[trip[:, 0], trip[:, 2], trip[:, 1]]
    lse_g = lse.cpu().numpy().astype(np.float64)[trip[:, 0], trip[:, 1], trip[:, 2]]
    check_fwd(o_g, lse_g, o_r, lse_r, "h32 hk8 sampled")
    dq_r, _ = oracle.attention_backward_rows_dq(q64, k64, v64, do64, trip, scale, 1)
    check_grad(to_f64(dq)[trip[:, 0], trip[:, 2], trip[:, 1]], dq_r, "h32 hk8 dq rows")
    dk_g, dv_g = to_f64(dk), to_f64(dv)
    for g in (0, 5):
        dk_r, dv_r = oracle.attention_backward_kv_head(q64, k64, v64, do64, 0, g, scale, 1)
        check_grad(dk_g[0, :, g], dk_r, f"dk kv head {g}")
        check_grad(dv_g[0, :, g], dv_r, f"dv kv head {g}")
