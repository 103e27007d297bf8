"""head_dim 256 backward (attn_bwd / attn_bwd_ex with D = 256): dQ, dK, dV from
the CUDA path (with the CUDA forward's O and LSE, as a training step would)
against the float64 oracle's analytic gradient on the same seeded inputs, at
the backward parity bars.  Sizes span several 128-row tiles and 64-wide steps
with ragged tails; causal, Sq != Sk in both directions, sliding windows,
grouped K/V heads, float16, and sampled rows of B1 H16 S8192 causal."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grad, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

D = 256


def _fwd_bwd(bits, causal, window, scale, fmt):
    import torch
    from exact_attention_156_b200 import attn_bwd, attn_fwd, get_last_device_error
    q, k, v, do = (to_device(bits[n], fmt) for n in ("q", "k", "v", "do"))
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=window)
    dq, dk, dv = attn_bwd(q, k, v, o, do, lse, softmax_scale=scale, causal=bool(causal),
                          window_size=window)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    return o, lse, dq, dk, dv


CASES = [
    # B, Sq, Sk, H, Hk, causal, window, fmt
    (1, 256, 256, 2, 2, 1, None, "bf16"),
    (1, 256, 256, 2, 2, 0, None, "bf16"),
    (2, 300, 457, 2, 2, 1, None, "bf16"),      # ragged, bottom-right causal
    (1, 457, 300, 2, 2, 1, None, "bf16"),      # Sq > Sk: early rows see no key
    (1, 520, 520, 2, 2, 1, (130, 0), "bf16"),  # sliding window
    (1, 333, 333, 3, 3, 0, (40, 25), "f16"),   # two-sided window, float16
    (2, 200, 333, 4, 2, 1, None, "f16"),       # grouped K/V heads, float16
    (1, 300, 300, 4, 1, 0, None, "bf16"),      # one K/V head for all query heads
    (1, 128, 128, 1, 1, 0, (0, 0), "bf16"),    # diagonal only
    (1, 1, 1, 1, 1, 0, None, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_d256_backward_full_tensor(case):
    B, Sq, Sk, H, Hk, causal, window, fmt = case
    bits = make_inputs(B, Sq, Sk, H, D, 7300 + Sq + 3 * Sk + H, 1.0, with_dout=True, Hk=Hk,
                       fmt=fmt)
    scale = 1.0 / np.sqrt(D)
    o, lse, dq, dk, dv = _fwd_bwd(bits, causal, window, scale, fmt)
    wl, wr = (-1, -1) if window is None else window
    ref = oracle.attention_backward(f64(bits["q"], fmt), f64(bits["k"], fmt), f64(bits["v"], fmt),
                                    f64(bits["do"], fmt), scale, causal, wl, wr)
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), ref["o"], ref["lse"], str(case))
    floor = 1e-3 * max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(to_f64(g), ref[name], f"{case} {name}", floor)


def test_d256_backward_sampled_b1h16s8192_causal():
    """The head_dim 256 workload (B1 H16 Sq=Sk=8192 causal, inputs N(0,1)*0.5):
    dQ on 2048 seeded (head, row) samples plus the first and last rows of every
    head; dK and dV on every key row of 2 seeded heads."""
    import torch
    B, S, H = 1, 8192, 16
    bits = make_inputs(B, S, S, H, D, 1009, 0.5, with_dout=True)
    scale = 1.0 / np.sqrt(D)
    o, lse, dq, dk, dv = _fwd_bwd(bits, 1, None, scale, "bf16")
    rng = np.random.default_rng(9)
    trip = np.stack([np.zeros(2048, dtype=np.int64), rng.integers(0, H, 2048),
                     rng.integers(0, S, 2048)], axis=1)
    edges = np.array([[0, h, r] for h in range(H) for r in (0, 1, S - 1)], dtype=np.int64)
    trip = np.unique(np.concatenate([trip, edges]), axis=0)
    t = torch.from_numpy(trip).cuda()
    wq, wk, wv, wdo = (f64(bits[n]) for n in ("q", "k", "v", "do"))
    dq_ref, _ = oracle.attention_backward_rows_dq(wq, wk, wv, wdo, trip, scale, 1)
    check_grad(to_f64(dq[t[:, 0], t[:, 2], t[:, 1]]), dq_ref, "d256 dq (sampled rows)")
    for h in np.random.default_rng(9).choice(H, size=2, replace=False):
        dk_ref, dv_ref = oracle.attention_backward_head(wq, wk, wv, wdo, 0, int(h), scale, 1)
        check_grad(to_f64(dk[0, :, int(h)]), dk_ref, f"d256 dk head {h}")
        check_grad(to_f64(dv[0, :, int(h)]), dv_ref, f"d256 dv head {h}")
