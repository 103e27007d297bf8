"""Padded batches (attn_fwd_padded / attn_bwd_padded): B sequences stored at
one padded length, each with its own real length.  The CUDA path against the
float64 oracle of the packed batch of the real rows (attention_forward_varlen
/ attention_backward_varlen), with the parity bars of the other tests; the
padding rows of every input hold NaN and +-inf (they must never be read), and
the padding rows of every output must come back as zeros (LSE -inf)."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grad, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu


def _poison(bits, lens, fmt):
    """Fill the padding rows of a (B, S, NH, D) 16-bit array with NaN / +-inf."""
    out = bits.copy()
    specials = ([0x7FC0, 0x7F80, 0xFF80] if fmt == "bf16" else [0x7E00, 0x7C00, 0xFC00])
    for b, n in enumerate(lens):
        pad = out[b, n:]
        pad[...] = np.array(specials, dtype=np.uint16)[np.arange(pad.size) % 3].reshape(pad.shape)
    return out


def _packed(bits, lens, fmt):
    """The real rows of a padded (B, S, NH, D) array, packed end to end (float64)."""
    return np.concatenate([f64(bits[b, :n], fmt) for b, n in enumerate(lens)], axis=0)


def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)


CASES = [
    # B, Sq, Sk, H, Hk, D, causal, window, fmt, lens_q, lens_k
    (3, 300, 300, 2, 2, 128, 1, None, "bf16", (300, 17, 211), (300, 17, 211)),
    (3, 257, 400, 4, 2, 64, 0, None, "f16", (257, 0, 130), (1, 399, 400)),
    (2, 200, 200, 2, 1, 128, 1, (50, 0), "bf16", (200, 129), (200, 129)),
    (4, 150, 150, 2, 2, 128, 1, None, "bf16", (0, 0, 150, 64), (0, 5, 150, 64)),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[:9]) for c in CASES])
def test_padded_forward_backward_against_the_oracle(case):
    import torch
    from exact_attention_156_b200 import (attn_bwd_padded, attn_fwd_padded,
                                          get_last_device_error)
    B, Sq, Sk, H, Hk, D, causal, window, fmt, lq, lk = case
    bits = make_inputs(B, Sq, Sk, H, D, 9100 + Sq + Sk + D, 1.0, with_dout=True, Hk=Hk, fmt=fmt)
    pq, pk, pv, pdo = (_poison(bits[n], lens, fmt)
                       for n, lens in (("q", lq), ("k", lk), ("v", lk), ("do", lq)))
    q, k, v, do = (to_device(x, fmt) for x in (pq, pk, pv, pdo))
    lens_q = torch.tensor(lq, dtype=torch.int32, device="cuda")
    lens_k = torch.tensor(lk, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_fwd_padded(q, k, v, lens_q, lens_k, softmax_scale=scale, causal=bool(causal),
                             window_size=window)
    dq, dk, dv = attn_bwd_padded(q, k, v, o, do, lse, lens_q, lens_k, softmax_scale=scale,
                                 causal=bool(causal), window_size=window)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    wl, wr = (-1, -1) if window is None else window
    ref = oracle.attention_backward_varlen(
        _packed(bits["q"], lq, fmt), _packed(bits["k"], lk, fmt), _packed(bits["v"], lk, fmt),
        _packed(bits["do"], lq, fmt), _cu(lq), _cu(lk), scale, causal, wl, wr)
    o_h, lse_h = to_f64(o), lse.cpu().numpy().astype(np.float64)
    dq_h, dk_h, dv_h = to_f64(dq), to_f64(dk), to_f64(dv)
    cq, ck = _cu(lq), _cu(lk)
    got_o = np.concatenate([o_h[b, :n] for b, n in enumerate(lq)])
    got_lse = np.concatenate([lse_h[b, :, :n] for b, n in enumerate(lq)], axis=1)
    check_fwd(got_o, got_lse.T, ref["o"], ref["lse"].T, f"{case[:9]} forward")
    floor = 1e-3 * max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for name, g, lens in (("dq", dq_h, lq), ("dk", dk_h, lk), ("dv", dv_h, lk)):
        got = np.concatenate([g[b, :n] for b, n in enumerate(lens)])
        check_grad(got, ref[name], f"{case[:9]} {name}", floor)
    # padding rows of every output: zeros, LSE -inf
    for b in range(B):
        assert not o_h[b, lq[b]:].any() and not dq_h[b, lq[b]:].any(), f"sequence {b}: q padding"
        assert not dk_h[b, lk[b]:].any() and not dv_h[b, lk[b]:].any(), f"sequence {b}: k padding"
        assert np.all(np.isneginf(lse_h[b, :, lq[b]:])), f"sequence {b}: LSE padding"
    assert cq[-1] == sum(lq) and ck[-1] == sum(lk)


def test_padded_rejects_bad_lengths_on_the_device():
    """A length outside [0, S] is reported (ATTN_ERR_SEQLENS) and that sequence
    reads as empty: its output rows are zeros, the others are unaffected."""
    import torch
    from exact_attention_156_b200 import attn_fwd, attn_fwd_padded, get_last_device_error
    B, S, H, D = 2, 256, 2, 128
    bits = make_inputs(B, S, S, H, D, 9200, 1.0)
    q, k, v = (to_device(bits[n]) for n in ("q", "k", "v"))
    lens = torch.tensor([S + 1, S], dtype=torch.int32, device="cuda")
    o, lse = attn_fwd_padded(q, k, v, lens, lens, causal=True)
    torch.cuda.synchronize()
    assert get_last_device_error() == 13  # ATTN_ERR_SEQLENS
    assert get_last_device_error() == 0   # read and cleared
    assert not to_f64(o[0]).any() and torch.isneginf(lse[0]).all()
    o1, lse1 = attn_fwd(q[1:], k[1:], v[1:], causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o[1], o1[0]) and torch.equal(lse[1], lse1[0])
