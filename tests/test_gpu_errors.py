"""Failure paths on the GPU that fault nothing: a bounded device-side wait that
runs out reports ATTN_ERR_TIMEOUT through the error word and the context stays
usable; bad pointers are refused on the host before any launch."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    import torch
    from exact_attention_156_b200 import attn_fwd, device_timeout_selftest, get_last_device_error
    assert get_last_device_error() == 0
    assert device_timeout_selftest(20000) == 0          # 20 ms limit on a barrier nobody completes
    assert get_last_device_error() == 9                 # ATTN_ERR_TIMEOUT, then cleared
    assert get_last_device_error() == 0
    # the context still runs real work afterwards
    q = torch.randn(1, 256, 2, 128, device="cuda").to(torch.bfloat16)
    o, lse = attn_fwd(q, q, q, causal=True)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    assert get_last_device_error() == 0


def test_host_pointer_is_refused():
    import torch
    from exact_attention_156_b200 import lib
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16, device="cuda")
    host = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16).pin_memory()
    lse = torch.zeros(1, 2, 128, dtype=torch.float32, device="cuda")
    st = lib.attn_fwd(host.data_ptr(), q.data_ptr(), q.data_ptr(), q.data_ptr(), lse.data_ptr(),
                      1, 128, 128, 2, 64, 0.125, 0, -1, -1, None)
    assert st == 7  # ATTN_ERR_DEVICE


def test_errors_leave_outputs_untouched():
    import torch
    from exact_attention_156_b200 import AttnError, attn_fwd
    q = torch.randn(1, 128, 2, 96, device="cuda").to(torch.bfloat16)
    with pytest.raises(AttnError, match="HEADDIM"):
        attn_fwd(q, q, q)
