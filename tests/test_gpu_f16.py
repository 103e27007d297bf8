"""IEEE float16 inputs (the _ex entry points with ATTN_DTYPE_F16): forward and
backward of the CUDA path against the float64 oracle evaluated on the same
float16-rounded values, with the parity bars of the bf16 tests."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grad, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # B, Sq, Sk, H, Hk, D, causal, wl, wr
    (1, 256, 256, 2, 2, 128, 1, -1, -1),
    (2, 300, 457, 2, 2, 64, 0, -1, -1),      # ragged, D = 64
    (1, 457, 300, 2, 2, 128, 1, -1, -1),     # Sq > Sk: rows that see nothing
    (1, 512, 512, 4, 1, 128, 1, 130, 0),     # multi-query with a sliding window
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_float16_forward_and_backward(case):
    import torch
    from exact_attention_156_b200 import (attn_bwd, attn_bwd_stages, attn_bwd_workspace_size,
                                          attn_fwd, get_last_device_error)
    B, Sq, Sk, H, Hk, D, causal, wl, wr = case
    bits = make_inputs(B, Sq, Sk, H, D, 4000 + sum(case), 1.0, with_dout=True, Hk=Hk, fmt="f16")
    q, k, v, do = (to_device(bits[n], "f16") for n in ("q", "k", "v", "do"))
    assert q.dtype == torch.float16
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=(wl, wr))
    assert o.dtype == torch.float16
    if B == 2:
        ws = torch.empty(attn_bwd_workspace_size(B, Sq, H, D), dtype=torch.uint8, device="cuda")
        dq, dk, dv = (torch.empty_like(x) for x in (q, k, v))
        attn_bwd_stages(q, k, v, o, do, lse, dq, dk, dv, ws, softmax_scale=scale,
                        causal=bool(causal), window_size=(wl, wr))
    else:
        dq, dk, dv = attn_bwd(q, k, v, o, do, lse, softmax_scale=scale, causal=bool(causal),
                              window_size=(wl, wr))
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    ref = oracle.attention_backward(f64(bits["q"], "f16"), f64(bits["k"], "f16"),
                                    f64(bits["v"], "f16"), f64(bits["do"], "f16"), scale, causal,
                                    wl, wr)
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), ref["o"], ref["lse"], str(case))
    floor = 1e-3 * max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        assert g.dtype == torch.float16
        check_grad(to_f64(g), ref[name], f"{case} {name}", floor)


def test_mixed_formats_are_refused():
    import torch
    from exact_attention_156_b200 import attn_fwd
    q = torch.zeros(1, 128, 2, 64, dtype=torch.float16, device="cuda")
    k = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(TypeError):
        attn_fwd(q, k, k)
