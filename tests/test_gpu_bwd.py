"""Backward parity: dQ, dK, dV from the CUDA path (using the CUDA forward's O
and LSE, as a training step would) against the float64 oracle's analytic
gradient on the same seeded inputs."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grad, f64, to_device, to_f64
from synth import bf16_bits_to_f32, config_by_name, make_config_inputs, make_inputs, sample_rows

pytestmark = pytest.mark.gpu


def _fwd_bwd(bits, causal, wl, wr, scale):
    import torch
    from exact_attention_156_b200 import attn_bwd, attn_fwd, get_last_device_error
    q, k, v, do = (to_device(bits[n]) for n in ("q", "k", "v", "do"))
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=(wl, wr))
    dq, dk, dv = attn_bwd(q, k, v, o, do, lse, softmax_scale=scale, causal=bool(causal),
                          window_size=(wl, wr))
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    return o, lse, dq, dk, dv


BWD_CASES = [
    # B, Sq, Sk, H, D, causal, wl, wr
    (1, 256, 256, 2, 128, 1, -1, -1),
    (1, 256, 256, 2, 128, 0, -1, -1),
    (2, 300, 457, 2, 128, 1, -1, -1),     # ragged, bottom-right causal
    (2, 300, 457, 2, 64, 0, -1, -1),
    (1, 457, 300, 2, 128, 1, -1, -1),     # Sq > Sk: rows that see nothing
    (1, 640, 640, 2, 128, 1, 130, 0),     # sliding window
    (1, 300, 300, 3, 64, 0, 40, 25),      # two-sided window, D = 64
    (1, 128, 128, 1, 128, 0, 0, 0),       # diagonal only
    (1, 1, 1, 1, 64, 0, -1, -1),
    (48, 70, 90, 2, 128, 1, -1, -1),      # many short problems (tile-major block order)
]


@pytest.mark.parametrize("case", BWD_CASES, ids=[str(c) for c in BWD_CASES])
def test_backward_full_tensor(case):
    B, Sq, Sk, H, D, causal, wl, wr = case
    bits = make_inputs(B, Sq, Sk, H, D, 2000 + sum(case), 1.0, with_dout=True)
    scale = 1.0 / np.sqrt(D)
    o, lse, dq, dk, dv = _fwd_bwd(bits, causal, wl, wr, scale)
    ref = oracle.attention_backward(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                    f64(bits["do"]), scale, causal, wl, wr)
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), ref["o"], ref["lse"], str(case))
    # floor: 1e-3 of the largest gradient magnitude of the problem
    floor = 1e-3 * max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(to_f64(g), ref[name], f"{case} {name}", floor)


def test_config_h32_s8192_fwd_bwd_sampled():
    """The fwd+bwd workload: dQ on >= 4096 sampled rows; dK and dV on every
    key row of 4 seeded heads (they sum over all query rows of the head)."""
    import torch
    cfg = config_by_name("c5")
    bits = make_config_inputs(cfg, with_dout=True)
    o, lse, dq, dk, dv = _fwd_bwd(bits, 1, -1, -1, cfg.scale)
    trip = sample_rows(cfg, 4096, 7)
    t = torch.from_numpy(trip).cuda()
    dq_s = to_f64(dq[t[:, 0], t[:, 2], t[:, 1]])
    o_s = to_f64(o[t[:, 0], t[:, 2], t[:, 1]])
    lse_s = lse[t[:, 0], t[:, 1], t[:, 2]].cpu().numpy().astype(np.float64)
    wq, wk, wv, wdo = (bf16_bits_to_f32(bits[n]) for n in ("q", "k", "v", "do"))
    o_ref, lse_ref = oracle.attention_forward_rows(wq, wk, wv, trip, cfg.scale, 1)
    check_fwd(o_s, lse_s, o_ref, lse_ref, "c5 forward")
    dq_ref, _ = oracle.attention_backward_rows_dq(wq, wk, wv, wdo, trip, cfg.scale, 1)
    # normalise by the largest dQ magnitude over the sampled rows
    check_grad(dq_s, dq_ref, "c5 dq (sampled rows)")
    heads = np.random.default_rng(7).choice(cfg.H, size=4, replace=False)
    for h in heads:
        dk_ref, dv_ref = oracle.attention_backward_head(wq, wk, wv, wdo, 0, int(h), cfg.scale, 1)
        check_grad(to_f64(dk[0, :, int(h)]), dk_ref, f"c5 dk head {h}")
        check_grad(to_f64(dv[0, :, int(h)]), dv_ref, f"c5 dv head {h}")
