"""head_dim 256 forward (attn_fwd / attn_fwd_ex with D = 256): the CUDA path
against the float64 oracle on the same seeded inputs, with the forward parity
bars.  Sizes span several 128-row query tiles and 64-key K/V tiles with ragged
tails; causal, Sq != Sk, grouped K/V heads, a sliding window, float16, and
sampled rows of a long sequence."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # B, Sq, Sk, H, Hk, causal, window, fmt
    (1, 300, 300, 2, 2, 1, None, "bf16"),
    (2, 200, 333, 4, 2, 0, None, "f16"),
    (1, 513, 513, 2, 1, 1, (64, 0), "bf16"),
    (2, 129, 65, 2, 2, 1, None, "bf16"),       # fewer keys than rows: early rows see none
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_d256_forward_against_the_oracle(case):
    import torch
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    B, Sq, Sk, H, Hk, causal, window, fmt = case
    D = 256
    bits = make_inputs(B, Sq, Sk, H, D, 7000 + Sq + Sk + H, 1.0, Hk=Hk, fmt=fmt)
    q, k, v = (to_device(bits[n], fmt) for n in ("q", "k", "v"))
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=bool(causal), window_size=window)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    wl, wr = (-1, -1) if window is None else window
    o_ref, lse_ref = oracle.attention_forward(f64(bits["q"], fmt), f64(bits["k"], fmt),
                                              f64(bits["v"], fmt), scale, causal, wl, wr)
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), o_ref, lse_ref, str(case))


def test_d256_sampled_rows_long_causal():
    """B1 H8 S4096 causal: 2048 seeded (head, row) samples plus the first and
    last rows of every head, against the oracle row by row."""
    import torch
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    B, S, H, D = 1, 4096, 8, 256
    bits = make_inputs(B, S, S, H, D, 7100, 0.5)
    q, k, v = (to_device(bits[n]) for n in ("q", "k", "v"))
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=True)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    rng = np.random.default_rng(8)
    trip = np.stack([np.zeros(2048, dtype=np.int64), rng.integers(0, H, 2048),
                     rng.integers(0, S, 2048)], axis=1)
    edges = np.array([[0, h, r] for h in range(H) for r in (0, 1, S - 1)], dtype=np.int64)
    trip = np.unique(np.concatenate([trip, edges]), axis=0)
    o_ref, lse_ref = oracle.attention_forward_rows(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                                   trip, scale, 1)
    o_d = to_f64(o)[trip[:, 0], trip[:, 2], trip[:, 1]]
    l_d = lse.cpu().numpy().astype(np.float64)[trip[:, 0], trip[:, 1], trip[:, 2]]
    check_fwd(o_d, l_d, o_ref, lse_ref, "d256 sampled rows")


def test_d256_bench_workload_sampled_rows():
    """The benchmark's head_dim 256 workload itself (B1 H16 Sq=Sk=8192 causal,
    its seed and scale), 1024 seeded (head, row) samples plus the first and last
    rows of every head, against the oracle row by row."""
    import torch
    import bench
    from exact_attention_156_b200 import attn_fwd, get_last_device_error
    w = bench.D256_WORKLOAD
    B, S, H, D = w["B"], w["Sq"], w["H"], w["D"]
    bits = make_inputs(B, S, S, H, D, w["seed"], w["input_scale"], Hk=w["Hk"])
    q, k, v = (to_device(bits[n]) for n in ("q", "k", "v"))
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_fwd(q, k, v, softmax_scale=scale, causal=True)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    rng = np.random.default_rng(9)
    trip = np.stack([np.zeros(1024, dtype=np.int64), rng.integers(0, H, 1024),
                     rng.integers(0, S, 1024)], axis=1)
    edges = np.array([[0, h, r] for h in range(H) for r in (0, S - 1)], dtype=np.int64)
    trip = np.unique(np.concatenate([trip, edges]), axis=0)
    o_ref, lse_ref = oracle.attention_forward_rows(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                                   trip, scale, 1)
    o_d = to_f64(o)[trip[:, 0], trip[:, 2], trip[:, 1]]
    l_d = lse.cpu().numpy().astype(np.float64)[trip[:, 0], trip[:, 1], trip[:, 2]]
    check_fwd(o_d, l_d, o_ref, lse_ref, "d256 bench workload rows")
