"""KV-cache decode (attn_decode): the CUDA path against the float64 oracle's
attention_decode on the same seeded inputs, with the forward parity bars.
Cases with at most 16 query rows per K/V head run the keys-on-lanes kernel,
the others the rows-on-lanes kernel; both at head_dim 64 and 128.
Cache rows past each sequence's length are filled with NaN and huge values:
they must not reach the result."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, f64, to_device, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # B, Sq, Smax, H, Hk, D, causal, lengths, fmt
    (2, 1, 1000, 8, 2, 128, 0, (1000, 333), "bf16"),
    (3, 4, 1024, 4, 4, 64, 1, (7, 513, 1024), "bf16"),
    (1, 2, 4096, 16, 1, 128, 1, (4000,), "bf16"),          # multi-query, two new rows
    (2, 1, 8192, 32, 8, 128, 0, (8192, 5000), "f16"),
    (2, 3, 300, 4, 2, 128, 1, (2, 300), "bf16"),           # a row that sees no key (L < Sq)
    (3, 1, 640, 8, 8, 64, 0, (0, 129, 640), "bf16"),       # an empty cache, one row past a tile
    (2, 1, 2048, 16, 1, 128, 0, (2048, 1500), "bf16"),     # 16 query heads on one K/V head
    (3, 1, 777, 4, 4, 128, 1, (777, 1, 129), "f16"),       # one row per K/V head, a one-key cache
    (1, 8, 1024, 2, 1, 128, 1, (1000,), "bf16"),           # 8 new positions x 2 heads, causal
    (2, 2, 1024, 16, 1, 64, 1, (1000, 77), "bf16"),        # 32 rows per K/V head: rows on the lanes
    (2, 1, 2048, 16, 1, 64, 0, (2048, 1500), "f16"),       # head_dim 64, 16 query heads on one
    (2, 5, 600, 6, 2, 64, 1, (3, 600), "bf16"),            # 15 rows per K/V head, L < Sq
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_decode_against_the_oracle(case):
    import torch
    from exact_attention_156_b200 import attn_decode, get_last_device_error
    B, Sq, Smax, H, Hk, D, causal, lens, fmt = case
    bits = make_inputs(B, Sq, Smax, H, D, 5000 + sum(case[:6]), 1.0, Hk=Hk, fmt=fmt)
    q, k, v = (to_device(bits[n], fmt) for n in ("q", "k", "v"))
    for b, L in enumerate(lens):          # stale, non-finite cache tail
        k[b, L:] = float("inf")
        v[b, L:] = float("nan")
    seqlens = torch.tensor(lens, dtype=torch.int32, device="cuda")
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_decode(q, k, v, seqlens, softmax_scale=scale, causal=bool(causal))
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    o_ref, lse_ref = oracle.attention_decode(f64(bits["q"], fmt), f64(bits["k"], fmt),
                                             f64(bits["v"], fmt), lens, scale, causal)
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), o_ref, lse_ref, str(case))


@pytest.mark.parametrize("name", ["DECODE_WORKLOAD", "DECODE64_WORKLOAD", "DECODE_ROWS_WORKLOAD"])
def test_decode_bench_workload_in_full(name):
    """The benchmark's decode workloads themselves (B8, one new row, H32 Hk8,
    8192 cached rows, D128 or D64; and four causal new rows of 32 query heads on
    one K/V head over 32768 cached rows; inputs N(0,1)*0.5, the seeds bench.py
    uses), every output row against the oracle, through the same call the
    benchmark times."""
    import torch
    import bench
    from exact_attention_156_b200 import (attn_decode, attn_decode_workspace_size,
                                          get_last_device_error)
    w = getattr(bench, name)
    B, Sq, H, Hk, S, D = w["B"], w["Sq"], w["H"], w["Hk"], w["Smax"], w["D"]
    bits = make_inputs(B, Sq, S, H, D, w["seed"], w["input_scale"], Hk=Hk)
    q, k, v = (to_device(bits[n]) for n in ("q", "k", "v"))
    seqlens = torch.full((B,), S, dtype=torch.int32, device="cuda")
    ws = torch.empty(attn_decode_workspace_size(B, Sq, S, H, Hk, D), dtype=torch.uint8,
                     device="cuda")
    o, lse = attn_decode(q, k, v, seqlens, causal=bool(w["causal"]), workspace=ws)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    o_ref, lse_ref = oracle.attention_decode(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                             [S] * B, 1.0 / np.sqrt(D), w["causal"])
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64), o_ref, lse_ref,
              f"decode bench workload {w['name']}")
