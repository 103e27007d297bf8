"""Forward parity: the CUDA kernel against the float64 oracle on the same
seeded bf16 inputs.  Small cases compare every element; the long workloads
compare >= 4096 seeded (batch, head, row) triples plus the causal edge rows."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, f64, to_device, to_f64
from synth import config_by_name, make_config_inputs, make_inputs, sample_rows

pytestmark = pytest.mark.gpu


def _run_dev(bits, causal, wl, wr, scale=None):
    import torch
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    q, k, v = (to_device(bits[n]) for n in ("q", "k", "v"))
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=(wl, wr))
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    return o, lse


def _run(bits, causal, wl, wr, scale=None):
    o, lse = _run_dev(bits, causal, wl, wr, scale)
    return to_f64(o), lse.cpu().numpy().astype(np.float64)


def _full_check(B, Sq, Sk, H, D, causal, wl, wr, seed, scale_in=1.0, q_mul=1.0, what=""):
    bits = make_inputs(B, Sq, Sk, H, D, seed, scale_in)
    if q_mul != 1.0:
        from synth import f32_to_bf16_bits, bf16_bits_to_f32
        bits["q"] = f32_to_bf16_bits(bf16_bits_to_f32(bits["q"]) * np.float32(q_mul))
    scale = 1.0 / np.sqrt(D)
    o, lse = _run(bits, causal, wl, wr, scale)
    o_ref, lse_ref = oracle.attention_forward(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                              scale, causal, wl, wr)
    return check_fwd(o, lse, o_ref, lse_ref, what)


def test_config_small_noncausal_d64():
    c = config_by_name("c1")
    _full_check(c.B, c.Sq, c.Sk, c.H, c.D, 0, -1, -1, c.seed, c.input_scale, what=c.name)


def test_config_b2_h16_s2048_causal_full_tensor():
    c = config_by_name("c2")
    _full_check(c.B, c.Sq, c.Sk, c.H, c.D, 1, -1, -1, c.seed, c.input_scale, what=c.name)


def test_peaked_scores_stress_rescaling():
    """Q x 8 makes the softmax peaked, so the running max moves by more than
    the rescale threshold many times along a row."""
    _full_check(2, 2048, 2048, 4, 128, 1, -1, -1, 77, 1.0, q_mul=8.0, what="peaked")


EDGE = [
    # B, Sq, Sk, H, D, causal, wl, wr
    (2, 300, 457, 3, 128, 0, -1, -1),
    (2, 300, 457, 3, 128, 1, -1, -1),     # bottom-right causal, ragged tails
    (2, 300, 457, 3, 64, 1, 100, 0),      # causal sliding window
    (1, 300, 457, 2, 128, 0, 37, 45),     # two-sided window
    (1, 333, 200, 2, 128, 1, -1, -1),     # Sq > Sk: first 133 rows see nothing
    (1, 1, 1, 1, 128, 0, -1, -1),         # S = 1
    (1, 129, 1, 2, 64, 0, -1, -1),        # one key
    (1, 260, 260, 2, 128, 0, 0, 0),       # diagonal window: O = V
    (1, 1000, 1000, 4, 64, 1, -1, -1),    # D = 64, several tiles
    (1, 640, 640, 2, 128, 1, 130, 0),     # window crossing tile edges
    (2, 1100, 1100, 20, 128, 1, -1, -1),  # more CTAs than SMs
    (2, 700, 900, 40, 64, 0, 200, 100),   # 240 work tiles, window, Sq != Sk
    (3, 96, 96, 5, 128, 1, -1, -1),       # Sq smaller than one tile
    (300, 40, 40, 1, 64, 0, -1, -1),      # many tiny problems (pair-major block order)
]


@pytest.mark.parametrize("case", EDGE, ids=[str(c) for c in EDGE])
def test_edge_cases_full_tensor(case):
    B, Sq, Sk, H, D, causal, wl, wr = case
    _full_check(B, Sq, Sk, H, D, causal, wl, wr, seed=1000 + sum(case), what=str(case))


def _sampled(cfg, causal, wl, wr, extra_rows=()):
    bits = make_config_inputs(cfg, with_dout=False)
    import torch
    o, lse = _run_dev(bits, causal, wl, wr, cfg.scale)
    trip = sample_rows(cfg, 4096, 7, extra_rows)
    t = torch.from_numpy(trip).cuda()
    o_s = to_f64(o[t[:, 0], t[:, 2], t[:, 1]])
    lse_s = lse[t[:, 0], t[:, 1], t[:, 2]].cpu().numpy().astype(np.float64)
    del o, lse
    o_ref, lse_ref = oracle.attention_forward_rows(_widen(bits["q"]), _widen(bits["k"]),
                                                   _widen(bits["v"]), trip, cfg.scale,
                                                   causal, wl, wr)
    return check_fwd(o_s, lse_s, o_ref, lse_ref, f"{cfg.name} causal={causal} win=({wl},{wr})")


def _widen(bits):
    from synth import bf16_bits_to_f32
    return bf16_bits_to_f32(bits)


@pytest.mark.parametrize("causal", [1, 0])
def test_config_h32_s8192_sampled(causal):
    _sampled(config_by_name("c3"), causal, -1, -1)


@pytest.mark.parametrize("variant", [(1, 4096, 0), (1, -1, -1)])
def test_config_h32_s32768_sampled(variant):
    _sampled(config_by_name("c4"), *variant, extra_rows=(4095, 4096, 4097))
