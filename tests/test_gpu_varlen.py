"""Packed variable-length batches (attn_fwd_varlen / attn_bwd_varlen): the
CUDA path against the float64 oracle on the same seeded inputs, with the
forward and gradient parity bars.  Lengths are ragged (not multiples of the
128-row tiles), include empty sequences and sequences with fewer keys than
query rows, and the sequences are packed back to back so that every tile
boundary falls inside a neighbour."""
import numpy as np
import pytest

import oracle
from helpers import check_fwd, check_grad, f64, to_f64
from synth import make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    # lengths_q, lengths_k, H, Hk, D, causal, window, fmt
    ((1, 127, 300, 1000), None, 4, 4, 128, 1, None, "bf16"),
    ((200, 0, 513, 64), (300, 100, 513, 1), 8, 2, 64, 1, None, "bf16"),
    ((129, 77, 640), (129, 0, 700), 2, 2, 128, 0, (32, 16), "f16"),
    ("many", None, 4, 1, 128, 1, None, "bf16"),
    # more sequences than a compact grid takes: the grid of the longest sequence's tiles
    ("many300", None, 2, 2, 64, 1, None, "bf16"),
]


def _lengths(case):
    lq, lk = case[0], case[1]
    if lq == "many":  # 40 short sequences, a packed fine-tuning batch
        rng = np.random.default_rng(77)
        lq = tuple(int(x) for x in rng.integers(1, 300, size=40))
    elif lq == "many300":  # 300 sequences: above the 256 that get compact grids
        rng = np.random.default_rng(78)
        lq = tuple(int(x) for x in rng.integers(0, 200, size=300))
    return lq, (lq if lk is None else lk)


def _packed_inputs(lq, lk, H, Hk, D, fmt, seed):
    """One sequence of every total length, drawn with the seeded recipe, then cut."""
    tq, tk = sum(lq), sum(lk)
    bits = make_inputs(1, tq, tk, H, D, seed, 1.0, with_dout=True, Hk=Hk, fmt=fmt)
    return {n: bits[n][0] for n in ("q", "k", "v", "do")}  # (total, heads, D)


def _to_dev(bits, fmt):
    import torch
    dtype = torch.float16 if fmt == "f16" else torch.bfloat16
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype).cuda()


@pytest.mark.parametrize("case", CASES, ids=[str(c[0])[:20] + f"-{c[4]}-{c[7]}" for c in CASES])
def test_varlen_fwd_bwd_against_the_oracle(case):
    import torch
    from exact_attention_156_b200 import attn_bwd_varlen, attn_fwd_varlen, get_last_device_error
    _, _, H, Hk, D, causal, window, fmt = case
    lq, lk = _lengths(case)
    bits = _packed_inputs(lq, lk, H, Hk, D, fmt, 6000 + H + D)
    q, k, v, do = (_to_dev(bits[n], fmt) for n in ("q", "k", "v", "do"))
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    cu_q, cu_k = torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda()
    scale = 1.0 / np.sqrt(D)
    o, lse = attn_fwd_varlen(q, k, v, cu_q, cu_k, max(lq), max(max(lk), 1), softmax_scale=scale,
                             causal=bool(causal), window_size=window)
    dq, dk, dv = attn_bwd_varlen(q, k, v, o, do, lse, cu_q, cu_k, max(lq), max(max(lk), 1),
                                 softmax_scale=scale, causal=bool(causal), window_size=window)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    wl, wr = (-1, -1) if window is None else window
    ref = oracle.attention_backward_varlen(f64(bits["q"], fmt), f64(bits["k"], fmt),
                                           f64(bits["v"], fmt), f64(bits["do"], fmt), cq, ck,
                                           scale, causal, wl, wr)
    # LSE is (H, total_q); check_fwd compares rows, so put the packed row first
    check_fwd(to_f64(o), lse.cpu().numpy().astype(np.float64).T, ref["o"], ref["lse"].T,
              f"fwd {case[0]}")
    top = max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(to_f64(got), ref[name], f"{name} {case[0]}", floor=1e-3 * top)
    # keys of sequences without query rows, rows of sequences without keys: exactly zero
    for b in range(len(lq)):
        if lq[b] == 0:
            assert torch.count_nonzero(dk[ck[b]:ck[b + 1]]) == 0
            assert torch.count_nonzero(dv[ck[b]:ck[b + 1]]) == 0
        if lk[b] == 0:
            assert torch.count_nonzero(o[cq[b]:cq[b + 1]]) == 0
            assert torch.count_nonzero(dq[cq[b]:cq[b + 1]]) == 0


def test_malformed_boundaries_are_reported_and_skipped():
    """Boundaries past the end and a decreasing pair: those sequences are
    skipped (their rows and keys keep what they held), the valid one is
    computed, and the device error word reports the problem once."""
    import torch
    from exact_attention_156_b200 import (ATTN_STATUS, attn_bwd_varlen, attn_fwd_varlen,
                                          get_last_device_error)
    lq = (100, 50, 150)
    bits = _packed_inputs(lq, lq, 2, 2, 64, "bf16", 6100)
    q, k, v, do = (_to_dev(bits[n], "bf16") for n in ("q", "k", "v", "do"))
    good = np.array([0, 100, 150, 300], dtype=np.int32)
    # sequence 1 ends past the 300 rows, sequence 2 starts after it ends
    bad = np.array([0, 100, 400, 300], dtype=np.int32)
    cu_bad = torch.from_numpy(bad).cuda()
    sentinel = 7.0
    o = torch.full_like(q, sentinel)
    lse = torch.full((2, 300), sentinel, dtype=torch.float32, device="cuda")
    attn_fwd_varlen(q, k, v, cu_bad, cu_bad, 150, 150, causal=True, out=o, lse=lse)
    assert ATTN_STATUS[get_last_device_error()] == "ATTN_ERR_SEQLENS"
    assert get_last_device_error() == 0   # reading clears it
    ref_o, ref_lse = oracle.attention_forward_varlen(f64(bits["q"]), f64(bits["k"]),
                                                     f64(bits["v"]), good, good,
                                                     1.0 / np.sqrt(64), 1)
    check_fwd(to_f64(o[:100]), lse[:, :100].cpu().numpy().astype(np.float64).T, ref_o[:100],
              ref_lse[:, :100].T, "valid sequence beside malformed ones")
    assert torch.all(o[100:] == sentinel)
    assert torch.all(lse[:, 100:] == sentinel)
    cu_good = torch.from_numpy(good).cuda()
    o_ok, lse_ok = attn_fwd_varlen(q, k, v, cu_good, cu_good, 150, 150, causal=True)
    dq, dk, dv = (torch.full_like(t, sentinel) for t in (q, k, v))
    attn_bwd_varlen(q, k, v, o_ok, do, lse_ok, cu_bad, cu_bad, 150, 150, causal=True, dq=dq,
                    dk=dk, dv=dv)
    assert ATTN_STATUS[get_last_device_error()] == "ATTN_ERR_SEQLENS"
    ref = oracle.attention_backward_varlen(f64(bits["q"]), f64(bits["k"]), f64(bits["v"]),
                                           f64(bits["do"]), good, good, 1.0 / np.sqrt(64), 1)
    top = max(np.abs(ref[n][:100]).max() for n in ("dq", "dk", "dv"))
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        check_grad(to_f64(got[:100]), ref[name][:100], f"{name} of the valid sequence",
                   floor=1e-3 * top)
        assert torch.all(got[100:] == sentinel), f"{name} rows of malformed sequences written"


def test_varlen_bench_workload_sampled_sequences():
    """The benchmark's packed batch itself (32768 tokens, 31 sequences of
    138..3872, H32 D128 causal, its seed and scale), run whole through the calls
    the benchmark times; the longest, the shortest and a middle sequence are
    checked against the oracle on four heads each (sequences and heads are
    independent, so their rows, keys and gradients are exact references)."""
    import torch
    import bench
    from exact_attention_156_b200 import attn_bwd_varlen, attn_fwd_varlen, get_last_device_error
    w = bench.VARLEN_WORKLOAD
    lengths = bench.varlen_lengths(w)
    T, H, D = w["total"], w["H"], w["D"]
    bits = make_inputs(1, T, T, H, D, w["seed"], w["input_scale"], with_dout=True, Hk=w["Hk"])
    x = {n: bits[n][0] for n in ("q", "k", "v", "do")}
    q, k, v, do = (_to_dev(x[n], "bf16") for n in ("q", "k", "v", "do"))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cu_d = torch.from_numpy(cu).cuda()
    Lmax = max(lengths)
    o, lse = attn_fwd_varlen(q, k, v, cu_d, cu_d, Lmax, Lmax, causal=True)
    dq, dk, dv = attn_bwd_varlen(q, k, v, o, do, lse, cu_d, cu_d, Lmax, Lmax, causal=True)
    torch.cuda.synchronize()
    assert get_last_device_error() == 0
    order = np.argsort(lengths)
    picks = sorted({int(order[-1]), int(order[0]), int(order[len(order) // 2])})
    heads = [0, 9, 21, 31]
    o_h, lse_h = to_f64(o), lse.cpu().numpy().astype(np.float64)
    g_h = {n: to_f64(t) for n, t in (("dq", dq), ("dk", dk), ("dv", dv))}
    for bi in picks:
        a, z = int(cu[bi]), int(cu[bi + 1])
        for h in heads:
            sl = lambda arr: f64(arr[a:z, h:h + 1])
            ref = oracle.attention_backward_varlen(sl(x["q"]), sl(x["k"]), sl(x["v"]),
                                                   sl(x["do"]), [0, z - a], [0, z - a],
                                                   1.0 / np.sqrt(D), 1)
            what = f"sequence {bi} (length {z - a}) head {h}"
            check_fwd(o_h[a:z, h:h + 1], lse_h[h:h + 1, a:z].T, ref["o"], ref["lse"].T, what)
            top = max(np.abs(ref[n]).max() for n in ("dq", "dk", "dv"))
            for n in ("dq", "dk", "dv"):
                check_grad(g_h[n][a:z, h:h + 1], ref[n], f"{n} {what}", floor=1e-3 * top)
