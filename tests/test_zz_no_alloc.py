"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory (for example code running inside a host that owns every device
allocation, or a latency-critical loop where an allocation would implicitly
synchronise the device).  Its scratch is a fixed 64 MiB array built into the
library instead of a caller-provided workspace.

Checked through the C ABI against attn_bwd (the entry point with a caller
workspace) on two calls in a row with different inputs, so that anything the
first call leaves in the shared scratch would show up in the second.  This
file is named so that pytest collects it last."""
import ctypes

import numpy as np
import pytest

from helpers import check_grad, to_device, to_f64
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


@pytest.mark.parametrize("case", [(1, 1000, 1000, 4, 128, 1, -1, -1),
                                  (2, 300, 457, 3, 64, 0, 50, 20)])
def test_noalloc_matches_workspace_backward_on_consecutive_calls(case):
    import torch
    from exact_attention_156_b200 import attn_bwd, attn_fwd, get_last_device_error, lib
    B, Sq, Sk, H, D, causal, wl, wr = case
    scale = 1.0 / np.sqrt(D)
    stream = torch.cuda.current_stream().cuda_stream
    for call, seed in enumerate((500, 501)):
        bits = make_inputs(B, Sq, Sk, H, D, seed + sum(case), 1.0, with_dout=True)
        q, k, v, do = (to_device(bits[n]) for n in ("q", "k", "v", "do"))
        o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=(wl, wr))
        ref = attn_bwd(q, k, v, o, do, lse, softmax_scale=scale, causal=bool(causal),
                       window_size=(wl, wr))
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        st = _noalloc(lib, q, k, v, o, do, lse, dq, dk, dv, scale, causal, wl, wr, stream)
        assert st == 0, f"call {call}: status {st}"
        torch.cuda.synchronize()
        assert get_last_device_error() == 0
        refs = [to_f64(t) for t in ref]
        floor = 1e-3 * max(np.abs(r).max() for r in refs)
        for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), refs):
            check_grad(to_f64(got), want, f"call {call} {name}", floor)


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
