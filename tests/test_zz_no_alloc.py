"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (for example code running inside a host that owns every device
allocation, or a latency-critical loop where an allocation would implicitly
synchronise the device).  Its scratch is a fixed 64 MiB array built into the
library instead of a caller-provided workspace.

Checked through the C ABI on two calls in a row:
  * against the float64 oracle at the parity bars of every other backward test;
  * against attn_bwd (the entry point with a caller workspace) on the same
    inputs: dK and dV come from the same kernels with no atomics, so they must
    be bit-identical; dQ differs only in the order of the float32 reduce-adds,
    so it must agree to one rounding step of its 16-bit format.
The second call is a smaller problem than the first (fewer query rows with the
same 128-row padding, and a different head count), so rows the first call left
in the shared scratch sit exactly where the second call must re-initialise
them.  This file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest

import oracle
from helpers import check_grad, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

ATTN_ERR_SCRATCH = 11


def _noalloc(lib, q, k, v, o, do, lse, dq, dk, dv, scale, causal, wl, wr, stream):
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    return lib.attn_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                do.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(),
                                dv.data_ptr(), B, Sq, Sk, H, D, ctypes.c_float(scale),
                                causal, wl, wr, stream)


def _one_call(case, seed):
    import torch
    from exact_attention_156_b200 import attn_bwd, attn_fwd, get_last_device_error, lib
    B, Sq, Sk, H, D, causal, wl, wr = case
    scale = 1.0 / np.sqrt(D)
    stream = torch.cuda.current_stream().cuda_stream
    bits = make_inputs(B, Sq, Sk, H, D, seed, 1.0, with_dout=True)
    q, k, v, do = (to_device(bits[n]) for n in ("q", "k", "v", "do"))
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=(wl, wr))
    ws_grads = attn_bwd(q, k, v, o, do, lse, softmax_scale=scale, causal=bool(causal),
                        window_size=(wl, wr))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    st = _noalloc(lib, q, k, v, o, do, lse, dq, dk, dv, scale, causal, wl, wr, stream)
    assert st == 0, f"status {st}"
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    w = {n: f64(bits[n]) for n in bits}
    ref = oracle.attention_backward(w["q"], w["k"], w["v"], w["do"], scale, causal, wl, wr)
    return (dq, dk, dv), ws_grads, ref


# (B, Sq, Sk, H, D, causal, win_left, win_right); each pair runs in this order,
# the second problem smaller than the first with the same padded query length.
PAIRS = [
    ((1, 1000, 1000, 4, 128, 1, -1, -1), (1, 900, 1000, 3, 128, 1, -1, -1)),
    ((2, 300, 457, 3, 64, 0, 50, 20), (1, 260, 300, 2, 64, 0, -1, 7)),
    ((1, 300, 300, 2, 256, 1, -1, -1), (1, 257, 300, 1, 256, 1, 60, 0)),
]


@pytest.mark.parametrize("pair", PAIRS)
def test_noalloc_matches_oracle_and_workspace_backward_on_consecutive_calls(pair):
    import torch
    for call, case in enumerate(pair):
        got, ws, ref = _one_call(case, 500 + call + sum(case))
        refs = [ref["dq"], ref["dk"], ref["dv"]]
        floor = 1e-3 * max(np.abs(r).max() for r in refs)
        for name, g, want in zip(("dq", "dk", "dv"), got, refs):
            check_grad(to_f64(g), want, f"call {call} {name} vs oracle", floor)
        # same kernels, same inputs: dK and dV bit-identical to the workspace path
        assert torch.equal(got[1], ws[1]), f"call {call}: dk differs from attn_bwd"
        assert torch.equal(got[2], ws[2]), f"call {call}: dv differs from attn_bwd"
        # dQ: only the order of the float32 reduce-adds differs -> within one
        # rounding step (2^-8 relative for bf16) of each element
        a, b = to_f64(got[0]), to_f64(ws[0])
        tol = np.abs(b) * 2.0 ** -7 + 1e-6 * np.abs(b).max()
        bad = np.abs(a - b) > tol
        assert not bad.any(), (f"call {call}: dq differs from attn_bwd in {int(bad.sum())} "
                               f"elements, max {np.abs(a - b).max():.3e}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    import torch
    from exact_attention_156_b200 import lib
    # B=1, H=32, Sq=8192, D=128 needs ~130 MiB of backward scratch (> 64 MiB)
    B, S, H, D = 1, 8192, 32, 128
    assert lib.attn_bwd_workspace_size(B, S, H, D) > (64 << 20)
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    p = t.data_ptr()
    st = lib.attn_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, S, S, H, D, ctypes.c_float(0.088),
                              1, -1, -1, None)
    assert st == ATTN_ERR_SCRATCH
    from exact_attention_156_b200 import status_string
    assert "64 MiB" in status_string(st)
