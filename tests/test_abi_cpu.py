"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/attn.h declares, and rejects bad arguments before
touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")
LIB = os.path.join(ROOT, "exact_attention_156_b200", "libattn156.so")

OK, NULLPTR, SHAPE, HEADDIM, ALIGN, WINDOW, ARCH, DEVICE = 0, 1, 2, 3, 4, 5, 6, 7


def declared_functions():
    text = open(HEADER).read()
    names = re.findall(r"ATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text)
    assert names, "no declarations found"
    return names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(LIB)
    names = declared_functions()
    assert {"attn_fwd", "attn_bwd", "attn_bwd_workspace_size", "attn_status_string"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in attn.h but not exported"


def test_status_enum_matches_binding():
    from exact_attention_156_b200 import ATTN_STATUS
    text = open(HEADER).read()
    block = text[:text.index("} attn_status;")]
    block = block[block.rindex("typedef enum"):]
    enum = dict((int(v), k) for k, v in re.findall(r"(ATTN_\w+)\s*=\s*(\d+)", block))
    assert enum == ATTN_STATUS
    dtypes = re.search(r"typedef enum \{([^}]*)\} attn_dtype;", text).group(1)
    from exact_attention_156_b200._binding import ATTN_DTYPE_BF16, ATTN_DTYPE_F16
    assert dict(re.findall(r"(ATTN_DTYPE_\w+)\s*=\s*(\d+)", dtypes)) == {
        "ATTN_DTYPE_BF16": str(ATTN_DTYPE_BF16), "ATTN_DTYPE_F16": str(ATTN_DTYPE_F16)}


def test_status_strings():
    from exact_attention_156_b200 import status_string
    for s in range(14):
        assert status_string(s) and status_string(s) != "unknown status"
    assert status_string(99) == "unknown status"


def _fwd(lib, q=0x1000, k=0x2000, v=0x3000, o=0x4000, lse=0x5000, B=1, Sq=128, Sk=128, H=2,
         D=128, scale=0.125, causal=0, wl=-1, wr=-1):
    return lib.attn_fwd(q, k, v, o, lse, B, Sq, Sk, H, D, scale, causal, wl, wr, None)


def test_fwd_validation_order_and_codes():
    from exact_attention_156_b200 import lib
    assert _fwd(lib, q=None) == NULLPTR
    assert _fwd(lib, lse=None) == NULLPTR
    assert _fwd(lib, B=0) == SHAPE
    assert _fwd(lib, Sk=0) == SHAPE
    assert _fwd(lib, H=70000) == SHAPE
    assert _fwd(lib, Sq=1 << 20, H=32, D=128) == SHAPE       # 2^32 elements
    assert _fwd(lib, D=96) == HEADDIM
    assert _fwd(lib, D=512) == HEADDIM
    assert _fwd(lib, D=256) in (ARCH, DEVICE)   # head_dim 256 passes validation
    assert _fwd(lib, scale=0.0) == SHAPE
    assert _fwd(lib, scale=float("nan")) == SHAPE
    assert _fwd(lib, scale=float("inf")) == SHAPE
    assert _fwd(lib, wl=-2) == WINDOW
    assert _fwd(lib, wr=-5) == WINDOW
    assert _fwd(lib, q=0x1008) == ALIGN
    assert _fwd(lib, lse=0x5002) == ALIGN


def test_bwd_validation_and_workspace_size():
    from exact_attention_156_b200 import lib
    assert lib.attn_bwd_workspace_size(1, 128, 2, 64) == 128 * 2 * (64 * 4 + 8)
    assert lib.attn_bwd_workspace_size(1, 129, 2, 128) == 256 * 2 * (128 * 4 + 8)
    assert lib.attn_bwd_workspace_size(0, 128, 2, 64) == 0
    assert lib.attn_bwd_workspace_size(1, 128, 2, 80) == 0
    # head_dim 256: the same layout (float32 dQ rows, then the two row values)
    assert lib.attn_bwd_workspace_size(2, 200, 3, 256) == 2 * 3 * 256 * (256 * 4 + 8)
    p = [0x1000 * (i + 1) for i in range(9)]
    ws = lib.attn_bwd_workspace_size(1, 128, 2, 128)

    def bwd(ptrs=p, B=1, Sq=128, Sk=128, H=2, D=128, wsp=0x100000, wsz=ws, wl=-1):
        return lib.attn_bwd(*ptrs, B, Sq, Sk, H, D, 0.1, 1, wl, -1, wsp, wsz, None)

    assert bwd(ptrs=[None] + p[1:]) == NULLPTR
    assert bwd(B=0) == SHAPE
    assert bwd(D=32) == HEADDIM
    assert bwd(D=256) == 10                 # head_dim 256 needs a larger workspace
    ws256 = lib.attn_bwd_workspace_size(1, 128, 2, 256)
    assert bwd(D=256, wsz=ws256) in (ARCH, DEVICE)  # then passes validation
    assert bwd(D=512, wsz=ws256) == HEADDIM
    assert bwd(wl=-3) == WINDOW
    assert bwd(ptrs=p[:6] + [0x7004] + p[7:]) == ALIGN
    assert bwd(wsp=None) == 10
    assert bwd(wsp=0x100010) == 10          # not 256-byte aligned
    assert bwd(wsz=ws - 4) == 10


def test_valid_arguments_without_a_gpu_fail_on_device_checks():
    """With well-formed arguments the next gate is the device: on a machine
    without a B200 (or with pointers that are not device memory) the call
    must refuse rather than launch."""
    from exact_attention_156_b200 import lib
    assert _fwd(lib) in (ARCH, DEVICE)


def test_binding_refuses_cpu_tensors():
    import torch
    from exact_attention_156_b200 import attn_fwd
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        attn_fwd(q, q, q)


def test_extended_entry_points_validate_heads_and_dtype():
    from exact_attention_156_b200 import lib
    DTYPE = 12

    def fwd(H, Hk, D=128, dtype=0):
        return lib.attn_fwd_ex(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 1, 128, 128, H, Hk, D,
                               dtype, 0.125, 1, -1, -1, None)
    assert fwd(8, 0) == SHAPE
    assert fwd(8, 16) == SHAPE
    assert fwd(8, 3) == SHAPE
    assert fwd(6, 4) == SHAPE
    assert fwd(8, 2, D=96) == HEADDIM
    assert fwd(8, 2, dtype=2) == DTYPE
    assert fwd(8, 2, dtype=-1) == DTYPE
    for dtype in (0, 1):                     # well-formed: stops at the device checks
        assert fwd(8, 2, dtype=dtype) in (ARCH, DEVICE)
        assert fwd(8, 1, dtype=dtype) in (ARCH, DEVICE)
    p = [0x1000 * (i + 1) for i in range(9)]
    ws = lib.attn_bwd_workspace_size(1, 128, 8, 128)
    assert lib.attn_bwd_ex(*p, 1, 128, 128, 8, 3, 128, 0, 0.1, 1, -1, -1, 0x100000, ws,
                           None) == SHAPE
    assert lib.attn_bwd_ex(*p, 1, 128, 128, 8, 2, 128, 5, 0.1, 1, -1, -1, 0x100000, ws,
                           None) == DTYPE
    assert lib.attn_bwd_main_ex(*p[:6], 1, 128, 128, 8, 0, 128, 1, 0.1, 1, -1, -1, 0x100000, ws,
                                None) == SHAPE
    assert lib.attn_bwd_ex(*p, 1, 128, 128, 8, 2, 128, 1, 0.1, 1, -1, -1, None, ws, None) == 10
    assert lib.attn_bwd_preprocess_ex(*p[:3], 1, 128, 8, 128, 7, 0x100000, ws, None) == DTYPE
    assert lib.attn_bwd_dq_finalize_ex(p[0], 1, 128, 8, 128, 9, 0.1, 0x100000, ws, None) == DTYPE


def test_binding_checks_key_value_heads():
    from types import SimpleNamespace

    from exact_attention_156_b200._binding import _kv_heads
    t = lambda *shape: SimpleNamespace(shape=shape)
    assert _kv_heads(t(1, 8, 8, 64), t(1, 8, 8, 64), t(1, 8, 8, 64)) == 8
    assert _kv_heads(t(1, 8, 8, 64), t(1, 8, 2, 64), t(1, 8, 2, 64)) == 2
    for k, v in ((t(1, 8, 3, 64), t(1, 8, 3, 64)), (t(1, 8, 2, 64), t(1, 8, 4, 64))):
        with pytest.raises(ValueError):
            _kv_heads(t(1, 8, 8, 64), k, v)


def test_decode_validation():
    from exact_attention_156_b200 import lib
    ws = lib.attn_decode_workspace_size(2, 1, 1024, 8, 2, 128)
    assert ws > 0
    assert lib.attn_decode_workspace_size(2, 1, 1024, 8, 3, 128) == 0
    assert lib.attn_decode_workspace_size(2, 1, 1024, 8, 2, 96) == 0

    def dec(Sq=1, H=8, Hk=2, D=128, dtype=0, wsp=0x100000, wsz=ws, seq=0x9000):
        return lib.attn_decode(0x1000, 0x2000, 0x3000, seq, 0x5000, 0x6000, 2, Sq, 1024, H, Hk,
                               D, dtype, 0.1, 1, wsp, wsz, None)
    assert dec(seq=None) == NULLPTR
    assert dec(Hk=3) == SHAPE
    assert dec(Sq=33, H=8, Hk=2) == SHAPE     # 4 heads x 33 rows > one 128-row tile
    assert dec(D=80) == HEADDIM
    assert dec(dtype=3) == 12
    assert dec(seq=0x9002) == ALIGN
    assert dec(wsp=None) == 10
    assert dec(wsz=ws - 1) == 10
    assert dec() in (ARCH, DEVICE)


def test_varlen_validation_and_workspace_size():
    from exact_attention_156_b200 import lib
    # rows per head: total_q + 132 B rounded up to 4; fp32 dQ row + two row values each
    assert lib.attn_bwd_varlen_workspace_size(3, 1000, 2, 64) == 2 * 1396 * (64 * 4 + 8)
    assert lib.attn_bwd_varlen_workspace_size(1, 1, 1, 128) == 136 * (128 * 4 + 8)
    assert lib.attn_bwd_varlen_workspace_size(0, 1000, 2, 64) == 0
    assert lib.attn_bwd_varlen_workspace_size(2, 1000, 2, 96) == 0

    def fwd(cu_q=0x9000, cu_k=0xA000, B=2, tq=300, tk=400, mq=200, mk=250, H=4, Hk=2, D=128,
            dtype=0, q=0x1000, lse=0x6000, wl=-1):
        return lib.attn_fwd_varlen(q, 0x2000, 0x3000, cu_q, cu_k, 0x4000, lse, B, tq, tk, mq, mk,
                                   H, Hk, D, dtype, 0.1, 1, wl, -1, None)
    assert fwd(cu_q=None) == NULLPTR
    assert fwd(B=0) == SHAPE
    assert fwd(tq=0) == SHAPE
    assert fwd(mq=0) == SHAPE
    assert fwd(mq=301) == SHAPE          # a sequence cannot be longer than the batch
    assert fwd(mk=401) == SHAPE
    assert fwd(Hk=3) == SHAPE
    assert fwd(D=80) == HEADDIM
    assert fwd(wl=-3) == WINDOW
    assert fwd(dtype=2) == 12
    assert fwd(q=0x1008) == ALIGN
    assert fwd(cu_k=0xA002) == ALIGN
    assert fwd(lse=0x6001) == ALIGN
    assert fwd() in (ARCH, DEVICE)
    ws = lib.attn_bwd_varlen_workspace_size(2, 300, 4, 128)

    def bwd(wsp=0x100000, wsz=ws, cu_q=0x9000):
        return lib.attn_bwd_varlen(0x1000, 0x2000, 0x3000, 0x4000, 0x5000, 0x6000, cu_q, 0xA000,
                                   0x7000, 0x8000, 0xB000, 2, 300, 400, 200, 250, 4, 2, 128, 0,
                                   0.1, 1, -1, -1, wsp, wsz, None)
    assert bwd(cu_q=None) == NULLPTR
    assert bwd(wsp=None) == 10
    assert bwd(wsp=0x100080) == 10       # not 256-byte aligned
    assert bwd(wsz=ws - 1) == 10
    assert bwd() in (ARCH, DEVICE)


def test_binding_refuses_cpu_tensors_on_every_entry_point():
    """No entry point has a CPU path: CPU tensors are refused in the binding,
    before the library is called."""
    import torch
    from exact_attention_156_b200 import (attn_bwd, attn_bwd_varlen, attn_decode,
                                          attn_fwd_varlen)
    q4 = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16)
    q3 = torch.zeros(128, 2, 64, dtype=torch.bfloat16)
    lse2 = torch.zeros(2, 128, dtype=torch.float32)
    lse3 = torch.zeros(1, 2, 128, dtype=torch.float32)
    cu = torch.tensor([0, 128], dtype=torch.int32)
    seq = torch.tensor([128], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        attn_bwd(q4, q4, q4, q4, q4, lse3)
    with pytest.raises(ValueError, match="CUDA"):
        attn_fwd_varlen(q3, q3, q3, cu, cu, 128, 128)
    with pytest.raises(ValueError, match="CUDA"):
        attn_bwd_varlen(q3, q3, q3, q3, q3, lse2, cu, cu, 128, 128)
    with pytest.raises(ValueError, match="CUDA"):
        attn_decode(torch.zeros(1, 1, 2, 64, dtype=torch.bfloat16), q4, q4, seq)


def test_binding_rejects_mixed_or_unsupported_formats():
    import torch
    from exact_attention_156_b200 import attn_fwd
    q = torch.zeros(1, 128, 2, 64, dtype=torch.float32)
    with pytest.raises(TypeError, match="bfloat16 or torch.float16"):
        attn_fwd(q, q, q)


def test_binding_checks_varlen_boundaries_on_the_host():
    """cu_seqlens must be a CUDA int32 vector; the binding refuses anything
    else before the library (whose device-side checks handle the values)."""
    import torch
    from exact_attention_156_b200._binding import _check_cu
    with pytest.raises(ValueError, match="CUDA"):
        _check_cu(torch.zeros(3, dtype=torch.int32), "cu_seqlens_q")
    with pytest.raises(TypeError):
        _check_cu([0, 1, 2], "cu_seqlens_q")


def _plan(lib, B, Smax, Hk, sms):
    ns, tps = ctypes.c_int(), ctypes.c_int()
    st = lib.attn_decode_split_plan(B, Smax, Hk, sms, ctypes.byref(ns), ctypes.byref(tps))
    return st, ns.value, tps.value


def test_decode_split_plan():
    """The decode planner (host logic): splits cover the cache, have at least
    two tiles unless the cache has one, never exceed the split count the
    workspace is sized for, and minimise the stated cost; brute force over every
    split length for a range of shapes and SM counts."""
    import math
    lib = ctypes.CDLL(LIB)
    assert _plan(lib, 8, 8192, 8, 148) == (OK, 2, 32)        # the bench workload: 128 CTAs
    from exact_attention_156_b200 import decode_split_plan
    assert decode_split_plan(8, 8192, 8, 148) == (2, 32)
    assert _plan(lib, 0, 8192, 8, 148)[0] == SHAPE
    assert _plan(lib, 1, 8192, 8, 0)[0] == SHAPE
    assert lib.attn_decode_split_plan(1, 1, 1, 1, None, None) == NULLPTR
    for B in (1, 2, 3, 8, 16, 64):
        for Smax in (1, 127, 128, 129, 1000, 4096, 8192, 32768):
            for Hk in (1, 2, 8):
                for sms in (1, 132, 148):
                    st, ns, tps = _plan(lib, B, Smax, Hk, sms)
                    assert st == OK
                    tiles = math.ceil(Smax / 128)
                    assert ns * tps >= tiles and (ns - 1) * tps < tiles
                    assert tps >= (2 if tiles > 1 else 1)
                    max_splits = (tiles + 1) // 2 if tiles > 1 else 1
                    assert 1 <= ns <= max_splits
                    cost = lambda t: math.ceil(B * Hk * math.ceil(tiles / t) / sms) * (t + 3)
                    best = min(cost(t) for t in range(2 if tiles > 1 else 1, tiles + 1))
                    assert cost(tps) == best, (B, Smax, Hk, sms, ns, tps)


def test_padded_validation_and_workspace_size():
    from exact_attention_156_b200 import lib
    wsf = lib.attn_fwd_padded_workspace_size(2, 300, 400, 4, 2, 128)
    wsb = lib.attn_bwd_padded_workspace_size(2, 300, 400, 4, 2, 128)
    # the backward also holds dO, dQ, dK, dV and the packed backward's own workspace
    assert 0 < wsf < wsb
    assert wsb - wsf >= lib.attn_bwd_varlen_workspace_size(2, 600, 4, 128)
    assert lib.attn_fwd_padded_workspace_size(2, 300, 400, 4, 2, 256) == 0   # head_dim 256
    assert lib.attn_fwd_padded_workspace_size(2, 300, 400, 4, 3, 128) == 0   # Hk must divide H
    assert lib.attn_bwd_padded_workspace_size(0, 300, 400, 4, 2, 128) == 0
    p = [0x1000 * (i + 1) for i in range(11)]
    f = ctypes.c_float

    def fwd(ptrs=p[:7], D=128, Hk=2, ws=0x200000, wsz=wsf, dtype=0):
        return lib.attn_fwd_padded(*ptrs, 2, 300, 400, 4, Hk, D, dtype, f(0.1), 1, -1, -1, ws,
                                   wsz, None)

    def bwd(ptrs=p, D=128, ws=0x200000, wsz=wsb):
        return lib.attn_bwd_padded(*ptrs, 2, 300, 400, 4, 2, D, 0, f(0.1), 1, -1, -1, ws, wsz,
                                   None)

    assert fwd(ptrs=p[:3] + [None] + p[4:7]) == NULLPTR
    assert fwd(D=256) == HEADDIM
    assert fwd(Hk=3) == SHAPE
    assert fwd(dtype=7) == 12
    assert fwd(ptrs=p[:3] + [0x3002] + p[4:7]) == ALIGN     # seqlens not 4-byte aligned
    assert fwd(ws=0x200010) == 10
    assert fwd(wsz=wsf - 1) == 10
    assert fwd() in (ARCH, DEVICE)
    assert bwd(ptrs=p[:10] + [None]) == NULLPTR
    assert bwd(wsz=wsb - 256) == 10
    assert bwd() in (ARCH, DEVICE)
