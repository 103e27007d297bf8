"""ctypes binding of the C ABI in include/attn.h (argument marshalling only).

Every step of attention runs in the CUDA kernels of ``libattn156.so``; this
module only turns torch tensors into pointers, sizes and the current stream,
and turns status codes into exceptions.  There is no CPU path: if the library
is missing the import fails.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn156.so")

ATTN_STATUS = {
    0: "ATTN_OK", 1: "ATTN_ERR_NULLPTR", 2: "ATTN_ERR_SHAPE", 3: "ATTN_ERR_HEADDIM",
    4: "ATTN_ERR_ALIGN", 5: "ATTN_ERR_WINDOW", 6: "ATTN_ERR_ARCH", 7: "ATTN_ERR_DEVICE",
    8: "ATTN_ERR_LAUNCH", 9: "ATTN_ERR_TIMEOUT", 10: "ATTN_ERR_WORKSPACE",
    11: "ATTN_ERR_SCRATCH", 12: "ATTN_ERR_DTYPE", 13: "ATTN_ERR_SEQLENS",
}
ATTN_DTYPE_BF16, ATTN_DTYPE_F16 = 0, 1


class AttnError(RuntimeError):
    def __init__(self, status: int, func: str):
        self.status = status
        self.name = ATTN_STATUS.get(status, str(status))
        super().__init__(f"{func}: {self.name}: {status_string(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m exact_attention_156_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    lib.attn_fwd.restype = i
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i,
                             vp, sz, vp]
    lib.attn_bwd.restype = i
    lib.attn_bwd_preprocess.argtypes = [vp, vp, vp, i, i, i, i, vp, sz, vp]
    lib.attn_bwd_preprocess.restype = i
    lib.attn_bwd_main.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, sz, vp]
    lib.attn_bwd_main.restype = i
    lib.attn_bwd_dq_finalize.argtypes = [vp, i, i, i, i, f, vp, sz, vp]
    lib.attn_bwd_dq_finalize.restype = i
    lib.attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i, vp]
    lib.attn_fwd_ex.restype = i
    lib.attn_bwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i,
                                i, vp, sz, vp]
    lib.attn_bwd_ex.restype = i
    lib.attn_bwd_preprocess_ex.argtypes = [vp, vp, vp, i, i, i, i, i, vp, sz, vp]
    lib.attn_bwd_preprocess_ex.restype = i
    lib.attn_bwd_main_ex.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i, vp,
                                     sz, vp]
    lib.attn_bwd_main_ex.restype = i
    lib.attn_bwd_dq_finalize_ex.argtypes = [vp, i, i, i, i, i, f, vp, sz, vp]
    lib.attn_bwd_dq_finalize_ex.restype = i
    lib.attn_decode_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.attn_decode_workspace_size.restype = sz
    lib.attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, sz, vp]
    lib.attn_decode.restype = i
    lib.attn_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f,
                                    i, i, i, vp]
    lib.attn_fwd_varlen.restype = i
    lib.attn_bwd_varlen_workspace_size.argtypes = [i, i, i, i]
    lib.attn_bwd_varlen_workspace_size.restype = sz
    lib.attn_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                    i, i, i, f, i, i, i, vp, sz, vp]
    lib.attn_bwd_varlen.restype = i
    lib.attn_decode_split_plan.argtypes = [i, i, i, i, ctypes.POINTER(i), ctypes.POINTER(i)]
    lib.attn_decode_split_plan.restype = i
    lib.attn_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i,
                                     i, vp]
    lib.attn_bwd_noalloc.restype = i
    lib.attn_fwd_padded_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.attn_fwd_padded_workspace_size.restype = sz
    lib.attn_bwd_padded_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.attn_bwd_padded_workspace_size.restype = sz
    lib.attn_fwd_padded.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i,
                                    vp, sz, vp]
    lib.attn_fwd_padded.restype = i
    lib.attn_bwd_padded.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i,
                                    i, f, i, i, i, vp, sz, vp]
    lib.attn_bwd_padded.restype = i
    lib.attn_bwd_workspace_size.argtypes = [i, i, i, i]
    lib.attn_bwd_workspace_size.restype = sz
    lib.attn_status_string.argtypes = [i]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_get_last_device_error.argtypes = []
    lib.attn_get_last_device_error.restype = i
    lib.attn_device_timeout_selftest.argtypes = [i, vp]
    lib.attn_device_timeout_selftest.restype = i
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.attn_status_string(int(status)).decode()


def _stream_handle(stream, device) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def _check(t, name, dtype, ndim):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (batch, seqlen, nheads, head_dim)")


def _dtype_code(t) -> int:
    """attn_dtype of a bf16 or f16 tensor (the format every 16-bit tensor of a call shares)."""
    import torch
    dtype = getattr(t, "dtype", None)
    if dtype == torch.bfloat16:
        return ATTN_DTYPE_BF16
    if dtype == torch.float16:
        return ATTN_DTYPE_F16
    raise TypeError(f"tensors must be torch.bfloat16 or torch.float16, got {dtype}")


def _kv_heads(q, k, v):
    """K/V head count; fewer than q's heads selects grouped K/V heads (GQA/MQA)."""
    H, Hk = q.shape[2], k.shape[2]
    if v.shape[2] != Hk or Hk < 1 or H % Hk != 0:
        raise ValueError(f"k and v must have the same number of heads, dividing q's {H}: "
                         f"k {tuple(k.shape)}, v {tuple(v.shape)}")
    return Hk


def _scale(softmax_scale, D):
    return float(1.0 / math.sqrt(D)) if softmax_scale is None else float(softmax_scale)


def _window(causal, window_size):
    wl, wr = (-1, -1) if window_size is None else (int(window_size[0]), int(window_size[1]))
    return (1 if causal else 0), wl, wr


def attn_fwd(q, k, v, softmax_scale: Optional[float] = None, causal: bool = False,
             window_size: Optional[Tuple[int, int]] = None, out=None, lse=None,
             stream=None):
    """O, LSE = exact attention of q (B,Sq,H,D), k, v (B,Sk,Hk,D), all bf16 (or all
    float16) CUDA tensors.

    Hk = H is ordinary multi-head attention; Hk < H (a divisor of H) shares each
    K/V head among H/Hk consecutive query heads (GQA; MQA when Hk = 1).
    ``softmax_scale=None`` means 1/sqrt(D).  ``window_size=(left, right)`` with
    -1 for an unbounded side.  Returns (o bf16 (B,Sq,H,D), lse fp32 (B,H,Sq)).
    """
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype, 4)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype, 4)
    _check(lse, "lse", torch.float32, 3)
    c, wl, wr = _window(causal, window_size)
    Hk = _kv_heads(q, k, v)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Sq, Sk)
    tail = (_scale(softmax_scale, D), c, wl, wr, _stream_handle(stream, q.device))
    if Hk == H and dt == ATTN_DTYPE_BF16:
        st, name = lib.attn_fwd(*args, H, D, *tail), "attn_fwd"
    else:
        st, name = lib.attn_fwd_ex(*args, H, Hk, D, dt, *tail), "attn_fwd_ex"
    if st != 0:
        raise AttnError(st, name)
    return out, lse


def attn_bwd_workspace_size(B: int, Sq: int, H: int, D: int) -> int:
    return int(lib.attn_bwd_workspace_size(B, Sq, H, D))


def attn_bwd(q, k, v, out, dout, lse, softmax_scale: Optional[float] = None,
             causal: bool = False, window_size: Optional[Tuple[int, int]] = None,
             dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of exact attention given the forward's O and LSE and dO.

    ``workspace`` (a uint8 CUDA tensor of at least attn_bwd_workspace_size
    bytes) is allocated by torch when not given.  Returns (dq, dk, dv) bf16.
    """
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, n, q.dtype, 4)
    _check(lse, "lse", torch.float32, 3)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = attn_bwd_workspace_size(B, Sq, H, D)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    c, wl, wr = _window(causal, window_size)
    Hk = _kv_heads(q, k, v)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
            lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, Sq, Sk)
    tail = (_scale(softmax_scale, D), c, wl, wr, workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), _stream_handle(stream, q.device))
    if Hk == H and dt == ATTN_DTYPE_BF16:
        st, name = lib.attn_bwd(*args, H, D, *tail), "attn_bwd"
    else:
        st, name = lib.attn_bwd_ex(*args, H, Hk, D, dt, *tail), "attn_bwd_ex"
    if st != 0:
        raise AttnError(st, name)
    return dq, dk, dv


def attn_bwd_stages(q, k, v, out, dout, lse, dq, dk, dv, workspace,
                    softmax_scale: Optional[float] = None, causal: bool = False,
                    window_size: Optional[Tuple[int, int]] = None, stream=None, between=None):
    """attn_bwd as its three C-ABI stages (preprocess, main, dq finalize).

    ``between(i)`` is called before stage i (0, 1, 2) and after the last one
    (i = 3) with no arguments otherwise; callers use it to record timing events
    on the same stream.  All tensors must be preallocated.
    """
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    dt = _dtype_code(q)
    c, wl, wr = _window(causal, window_size)
    sc = _scale(softmax_scale, D)
    hs = _stream_handle(stream, q.device)
    wp, wb = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    Hk = _kv_heads(q, k, v)
    plain = Hk == H and dt == ATTN_DTYPE_BF16
    if between:
        between(0)
    if plain:
        st, name = lib.attn_bwd_preprocess(out.data_ptr(), dout.data_ptr(), lse.data_ptr(), B, Sq,
                                           H, D, wp, wb, hs), "attn_bwd_preprocess"
    else:
        st, name = lib.attn_bwd_preprocess_ex(out.data_ptr(), dout.data_ptr(), lse.data_ptr(), B,
                                              Sq, H, D, dt, wp, wb, hs), "attn_bwd_preprocess_ex"
    if st != 0:
        raise AttnError(st, name)
    if between:
        between(1)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), dout.data_ptr(), dk.data_ptr(),
            dv.data_ptr(), B, Sq, Sk)
    if plain:
        st, name = lib.attn_bwd_main(*args, H, D, sc, c, wl, wr, wp, wb, hs), "attn_bwd_main"
    else:
        st, name = (lib.attn_bwd_main_ex(*args, H, Hk, D, dt, sc, c, wl, wr, wp, wb, hs),
                    "attn_bwd_main_ex")
    if st != 0:
        raise AttnError(st, name)
    if between:
        between(2)
    if plain:
        st, name = lib.attn_bwd_dq_finalize(dq.data_ptr(), B, Sq, H, D, sc, wp, wb, hs), \
            "attn_bwd_dq_finalize"
    else:
        st, name = lib.attn_bwd_dq_finalize_ex(dq.data_ptr(), B, Sq, H, D, dt, sc, wp, wb, hs), \
            "attn_bwd_dq_finalize_ex"
    if st != 0:
        raise AttnError(st, name)
    if between:
        between(3)
    return dq, dk, dv


def attn_decode_workspace_size(B: int, Sq: int, Smax: int, H: int, Hk: int, D: int) -> int:
    return int(lib.attn_decode_workspace_size(B, Sq, Smax, H, Hk, D))


def decode_split_plan(B: int, Smax: int, Hk: int, num_sms: int):
    """(splits, tiles per split) attn_decode uses for this shape on a GPU with
    num_sms SMs (host logic; no device needed)."""
    ns, tps = ctypes.c_int(), ctypes.c_int()
    st = lib.attn_decode_split_plan(B, Smax, Hk, num_sms, ctypes.byref(ns), ctypes.byref(tps))
    if st != 0:
        raise AttnError(st, "attn_decode_split_plan")
    return ns.value, tps.value


def attn_decode(q, k_cache, v_cache, cache_seqlens, softmax_scale: Optional[float] = None,
                causal: bool = False, out=None, lse=None, workspace=None, stream=None):
    """Attention of the Sq newest query rows q (B,Sq,H,D) of each sequence over
    the first cache_seqlens[b] rows of k_cache, v_cache (B,Smax,Hk,D).

    cache_seqlens is an int32 CUDA tensor (B,).  All 16-bit tensors share one
    format (bf16 or float16).  Returns (o (B,Sq,H,D), lse fp32 (B,H,Sq)).
    """
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k_cache, "k_cache"), (v_cache, "v_cache")):
        _check(t, n, q.dtype, 4)
    _check(cache_seqlens, "cache_seqlens", torch.int32, 1)
    B, Sq, H, D = q.shape
    Smax = k_cache.shape[1]
    Hk = _kv_heads(q, k_cache, v_cache)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    need = attn_decode_workspace_size(B, Sq, Smax, H, Hk, D)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    st = lib.attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                         cache_seqlens.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Sq, Smax, H,
                         Hk, D, dt, _scale(softmax_scale, D), 1 if causal else 0,
                         workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                         _stream_handle(stream, q.device))
    if st != 0:
        raise AttnError(st, "attn_decode")
    return out, lse


def _check_cu(cu, name, B_plus_1=None):
    import torch
    _check(cu, name, torch.int32, 1)
    if cu.numel() < 2 or (B_plus_1 is not None and cu.numel() != B_plus_1):
        raise ValueError(f"{name} must hold batch + 1 >= 2 boundaries, got {cu.numel()}")


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    softmax_scale: Optional[float] = None, causal: bool = False,
                    window_size: Optional[Tuple[int, int]] = None, out=None, lse=None,
                    stream=None):
    """Exact attention of a batch of sequences of different lengths packed end
    to end: q (total_q, H, D), k, v (total_k, Hk, D); sequence b is rows
    cu_seqlens_q[b]:cu_seqlens_q[b+1] of q and cu_seqlens_k[b]:cu_seqlens_k[b+1]
    of k and v (int32 CUDA tensors of batch + 1 boundaries).  max_seqlen_q/_k
    bound the sequence lengths (host ints, as the caller knows them).  Returns
    (o (total_q, H, D), lse fp32 (H, total_q)).
    """
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype, 3)
    _check_cu(cu_seqlens_q, "cu_seqlens_q")
    _check_cu(cu_seqlens_k, "cu_seqlens_k", cu_seqlens_q.numel())
    total_q, H, D = q.shape
    total_k, Hk = k.shape[0], k.shape[1]
    if v.shape[1] != Hk or Hk < 1 or H % Hk != 0:
        raise ValueError(f"k and v must have the same number of heads, dividing q's {H}")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    _check(out, "out", q.dtype, 3)
    _check(lse, "lse", torch.float32, 2)
    c, wl, wr = _window(causal, window_size)
    st = lib.attn_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), cu_seqlens_q.data_ptr(),
                             cu_seqlens_k.data_ptr(), out.data_ptr(), lse.data_ptr(),
                             cu_seqlens_q.numel() - 1, total_q, total_k, int(max_seqlen_q),
                             int(max_seqlen_k), H, Hk, D, dt, _scale(softmax_scale, D), c, wl,
                             wr, _stream_handle(stream, q.device))
    if st != 0:
        raise AttnError(st, "attn_fwd_varlen")
    return out, lse


def attn_bwd_varlen_workspace_size(B: int, total_q: int, H: int, D: int) -> int:
    return int(lib.attn_bwd_varlen_workspace_size(B, total_q, H, D))


def attn_bwd_varlen(q, k, v, out, dout, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                    max_seqlen_k: int, softmax_scale: Optional[float] = None,
                    causal: bool = False, window_size: Optional[Tuple[int, int]] = None,
                    dq=None, dk=None, dv=None, workspace=None, stream=None):
    """dQ, dK, dV of ``attn_fwd_varlen`` (same packed layout) given its O and
    LSE and dO.  Returns (dq, dk, dv)."""
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, n, q.dtype, 3)
    _check(lse, "lse", torch.float32, 2)
    _check_cu(cu_seqlens_q, "cu_seqlens_q")
    _check_cu(cu_seqlens_k, "cu_seqlens_k", cu_seqlens_q.numel())
    total_q, H, D = q.shape
    total_k, Hk = k.shape[0], k.shape[1]
    if v.shape[1] != Hk or Hk < 1 or H % Hk != 0:
        raise ValueError(f"k and v must have the same number of heads, dividing q's {H}")
    B = cu_seqlens_q.numel() - 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(attn_bwd_varlen_workspace_size(B, total_q, H, D),
                                dtype=torch.uint8, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.attn_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             dout.data_ptr(), lse.data_ptr(), cu_seqlens_q.data_ptr(),
                             cu_seqlens_k.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                             B, total_q, total_k, int(max_seqlen_q), int(max_seqlen_k), H, Hk, D,
                             dt, _scale(softmax_scale, D), c, wl, wr, workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(),
                             _stream_handle(stream, q.device))
    if st != 0:
        raise AttnError(st, "attn_bwd_varlen")
    return dq, dk, dv


def attn_fwd_padded_workspace_size(B: int, Sq: int, Sk: int, H: int, Hk: int, D: int) -> int:
    return int(lib.attn_fwd_padded_workspace_size(B, Sq, Sk, H, Hk, D))


def attn_bwd_padded_workspace_size(B: int, Sq: int, Sk: int, H: int, Hk: int, D: int) -> int:
    return int(lib.attn_bwd_padded_workspace_size(B, Sq, Sk, H, Hk, D))


def _check_seqlens(t, name, B):
    import torch
    _check(t, name, torch.int32, 1)
    if t.numel() != B:
        raise ValueError(f"{name} must hold one length per sequence ({B}), got {t.numel()}")


def attn_fwd_padded(q, k, v, seqlens_q, seqlens_k, softmax_scale: Optional[float] = None,
                    causal: bool = False, window_size: Optional[Tuple[int, int]] = None,
                    out=None, lse=None, workspace=None, stream=None):
    """Exact attention of a padded batch: q (B, Sq, H, D), k, v (B, Sk, Hk, D);
    sequence b's real rows are its first seqlens_q[b] / seqlens_k[b] rows (int32
    CUDA tensors of B lengths).  Padding rows are never read; those of the
    output are zero and their LSE -inf.  Returns (o (B, Sq, H, D), lse (B, H, Sq))."""
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _check(t, n, q.dtype, 4)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    Hk = _kv_heads(q, k, v)
    _check_seqlens(seqlens_q, "seqlens_q", B)
    _check_seqlens(seqlens_k, "seqlens_k", B)
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device) if lse is None else lse
    _check(out, "out", q.dtype, 4)
    _check(lse, "lse", torch.float32, 3)
    if workspace is None:
        workspace = torch.empty(max(attn_fwd_padded_workspace_size(B, Sq, Sk, H, Hk, D), 256),
                                dtype=torch.uint8, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.attn_fwd_padded(q.data_ptr(), k.data_ptr(), v.data_ptr(), seqlens_q.data_ptr(),
                             seqlens_k.data_ptr(), out.data_ptr(), lse.data_ptr(), B, Sq, Sk, H,
                             Hk, D, dt, _scale(softmax_scale, D), c, wl, wr,
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_handle(stream, q.device))
    if st != 0:
        raise AttnError(st, "attn_fwd_padded")
    return out, lse


def attn_bwd_padded(q, k, v, out, dout, lse, seqlens_q, seqlens_k,
                    softmax_scale: Optional[float] = None, causal: bool = False,
                    window_size: Optional[Tuple[int, int]] = None, dq=None, dk=None, dv=None,
                    workspace=None, stream=None):
    """dQ, dK, dV of ``attn_fwd_padded`` (same padded layout) given its O and
    LSE and dO; padding rows of the gradients are zero.  Returns (dq, dk, dv)."""
    import torch
    dt = _dtype_code(q)
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (dout, "dout")):
        _check(t, n, q.dtype, 4)
    _check(lse, "lse", torch.float32, 3)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    Hk = _kv_heads(q, k, v)
    _check_seqlens(seqlens_q, "seqlens_q", B)
    _check_seqlens(seqlens_k, "seqlens_k", B)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(max(attn_bwd_padded_workspace_size(B, Sq, Sk, H, Hk, D), 256),
                                dtype=torch.uint8, device=q.device)
    c, wl, wr = _window(causal, window_size)
    st = lib.attn_bwd_padded(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                             dout.data_ptr(), lse.data_ptr(), seqlens_q.data_ptr(),
                             seqlens_k.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B,
                             Sq, Sk, H, Hk, D, dt, _scale(softmax_scale, D), c, wl, wr,
                             workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             _stream_handle(stream, q.device))
    if st != 0:
        raise AttnError(st, "attn_bwd_padded")
    return dq, dk, dv


def get_last_device_error() -> int:
    """Synchronises the device; returns the status a kernel recorded (a timed-out
    wait, malformed packed-sequence boundaries), 0 if none."""
    return int(lib.attn_get_last_device_error())


def device_timeout_selftest(limit_us: int, stream=None) -> int:
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    return int(lib.attn_device_timeout_selftest(int(limit_us), _stream_handle(stream, dev)))
