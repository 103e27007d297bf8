"""The benchmark's work and byte accounting (host logic, no GPU): the counts it
divides by must be the stated conventions — 4*B*H*Sq*Sk*D forward flops halved
for causal, 2.5x that for the backward, visible pairs for a window, K and V bytes
of every valid cache row for decode — checked against independent counts."""
import math

import numpy as np

import bench
from synth import packed_lengths


def test_headline_flops():
    w = bench.WORKLOAD
    assert math.isclose(bench.fwd_flops(w), 549.755813888e9, rel_tol=1e-12)
    assert math.isclose(bench.bwd_flops(w), 2.5 * 549.755813888e9, rel_tol=1e-12)
    assert math.isclose(bench.step_flops(w), 3.5 * 549.755813888e9, rel_tol=1e-12)


def test_visible_keys_against_a_mask_count():
    """visible_keys(i) equals the count of an explicit (i, j) mask on small
    shapes with causal, windows and Sq != Sk."""
    for (Sq, Sk, causal, wl, wr) in ((7, 7, 1, -1, -1), (5, 9, 1, 2, 0), (9, 5, 1, -1, -1),
                                     (6, 6, 0, 1, 2), (8, 8, 1, 0, 0)):
        w = dict(Sq=Sq, Sk=Sk, causal=causal, win_left=wl, win_right=wr)
        d = Sk - Sq
        for i in range(Sq):
            j = np.arange(Sk)
            vis = np.ones(Sk, dtype=bool)
            if causal:
                vis &= j <= i + d
            if wl >= 0:
                vis &= j >= i + d - wl
            if wr >= 0:
                vis &= j <= i + d + wr
            assert bench.visible_keys(i, w) == int(vis.sum()), (Sq, Sk, causal, wl, wr, i)


def test_window_workload_visible_pairs():
    """Causal with window (4096, 0) at 32768: rows see min(i, 4096) + 1 keys,
    125,859,840 pairs per head in all (the count the work is reported on)."""
    w = dict(Sq=32768, Sk=32768, causal=1, win_left=4096, win_right=0)
    pairs = sum(bench.visible_keys(i, w) for i in range(32768))
    assert pairs == sum(min(i, 4096) + 1 for i in range(32768)) == 125_859_840
    assert math.isclose(4 * 128 * pairs * 32, 2062.09e9, rel_tol=1e-5)


def test_decode_bytes():
    w = bench.DECODE_WORKLOAD
    kv = 2 * w["B"] * w["Smax"] * w["Hk"] * w["D"] * 2
    qo = 2 * w["B"] * w["Sq"] * w["H"] * w["D"] * 2
    assert bench.decode_bytes(w) == kv + qo == 268_566_528


def test_varlen_accounting_and_lengths():
    w = bench.VARLEN_WORKLOAD
    lengths = bench.varlen_lengths(w)
    assert sum(lengths) == w["total"]
    assert all(w["len_lo"] <= L <= w["len_hi"] for L in lengths[:-1])
    assert 1 <= lengths[-1] <= w["len_hi"]
    assert lengths == packed_lengths(w["total"], w["len_lo"], w["len_hi"], w["seed"])
    f = bench.varlen_fwd_flops(w, lengths)
    assert math.isclose(f, sum(4.0 * w["H"] * L * L * w["D"] / 2 for L in lengths))
    # one sequence of the whole batch would be the dense count
    assert math.isclose(bench.varlen_fwd_flops(w, (w["total"],)),
                        bench.fwd_flops(dict(B=1, H=w["H"], Sq=w["total"], Sk=w["total"],
                                             D=w["D"], causal=1)))


def test_packed_lengths_edge_cases():
    assert packed_lengths(10, 100, 200, 1) == (10,)          # first draw cut to fit
    assert sum(packed_lengths(1000, 1, 1, 3)) == 1000        # all ones
    assert packed_lengths(1000, 16, 64, 5) == packed_lengths(1000, 16, 64, 5)
