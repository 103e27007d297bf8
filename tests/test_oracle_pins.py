"""Pins for the float64 oracle: closed forms, invariants, brute force and
finite differences.  None of these re-types the oracle's formula; each is a
fact the definition of attention implies and that a plausible slip in the
oracle (dropped term, wrong sign or index, transposed operand, wrong mask
bound, wrong normaliser) would break.
"""
import math

import numpy as np
import pytest

from oracle import (attention_backward, attention_backward_head,
                    attention_backward_rows_dq, attention_forward,
                    attention_forward_rows, online_softmax_forward)

MASKS = [
    # (Sq, Sk, causal, win_left, win_right)
    (7, 7, 0, -1, -1),
    (7, 7, 1, -1, -1),
    (5, 9, 1, -1, -1),     # Sq < Sk: bottom-right causal
    (9, 5, 1, -1, -1),     # Sq > Sk: first rows see nothing
    (11, 11, 1, 3, 0),     # sliding window, causal
    (11, 11, 0, 2, 1),     # two-sided window
    (8, 13, 0, 0, 0),      # diagonal only (shifted by Sk - Sq)
    (6, 6, 0, -1, 2),
]


def _bounds(i, Sq, Sk, causal, wl, wr):
    """Inclusive visible key range of query i, from the stated mask reading."""
    d = Sk - Sq
    lo, hi = 0, Sk - 1
    if causal:
        hi = min(hi, i + d)
    if wl >= 0:
        lo = max(lo, i + d - wl)
    if wr >= 0:
        hi = min(hi, i + d + wr)
    return lo, hi


def _rand(rng, *shape):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("mask", MASKS)
def test_zero_query_gives_mean_of_visible_values(mask):
    """Q = 0 makes every visible score 0: O_i is the plain mean of the visible
    V rows and LSE_i = ln(#visible); rows with nothing visible give 0, -inf."""
    Sq, Sk, causal, wl, wr = mask
    rng = np.random.default_rng(1)
    B, H, D = 2, 3, 5
    q = np.zeros((B, Sq, H, D))
    k = _rand(rng, B, Sk, H, D)
    v = _rand(rng, B, Sk, H, D)
    o, lse = attention_forward(q, k, v, 0.37, causal, wl, wr)
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                lo, hi = _bounds(i, Sq, Sk, causal, wl, wr)
                if hi < lo:
                    assert np.all(o[b, i, h] == 0.0)
                    assert lse[b, h, i] == -np.inf
                    continue
                n = hi - lo + 1
                acc = np.zeros(D)
                for j in range(lo, hi + 1):
                    acc += v[b, j, h]
                np.testing.assert_allclose(o[b, i, h], acc / n, rtol=1e-13, atol=1e-14)
                assert abs(lse[b, h, i] - math.log(n)) < 1e-13


@pytest.mark.parametrize("causal", [0, 1])
def test_single_dominant_score_selects_that_value_row(causal):
    """If score (i, j*) exceeds all others by ~60, O_i = V_j* and LSE_i = S_ij*
    to within exp(-60)."""
    rng = np.random.default_rng(2)
    S, D, scale = 10, 12, 0.5
    k = _rand(rng, 1, S, 1, D)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = _rand(rng, 1, S, 1, D)
    q = np.zeros((1, S, 1, D))
    targets = []
    for i in range(S):
        js = int(rng.integers(0, i + 1)) if causal else int(rng.integers(0, S))
        # choose q_i along the component of k_js orthogonal to the other keys' span
        others = [j for j in range(S) if j != js and (not causal or j <= i)]
        kj = k[0, js, 0].copy()
        if others:
            A = k[0, others, 0].T
            coef, *_ = np.linalg.lstsq(A, kj, rcond=None)
            kj = kj - A @ coef
        # make scale * q . k_js = 60 and scale * q . k_other = 0
        q[0, i, 0] = kj * (60.0 / (scale * float(kj @ k[0, js, 0])))
        targets.append(js)
    o, lse = attention_forward(q, k, v, scale, causal)
    for i, js in enumerate(targets):
        np.testing.assert_allclose(o[0, i, 0], v[0, js, 0], rtol=0, atol=1e-20)
        assert abs(lse[0, 0, i] - 60.0) < 1e-12


def test_joint_permutation_of_keys_and_values_is_invisible():
    """Non-causal attention is a function of the set of (k_j, v_j) pairs."""
    rng = np.random.default_rng(3)
    B, Sq, Sk, H, D = 2, 9, 13, 2, 7
    q, k, v = _rand(rng, B, Sq, H, D), _rand(rng, B, Sk, H, D), _rand(rng, B, Sk, H, D)
    perm = rng.permutation(Sk)
    o1, l1 = attention_forward(q, k, v, 0.4)
    o2, l2 = attention_forward(q, k[:, perm], v[:, perm], 0.4)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-13)
    # negative control: permuting V alone must change the output
    o3, _ = attention_forward(q, k, v[:, perm], 0.4)
    assert np.max(np.abs(o3 - o1)) > 1e-3


@pytest.mark.parametrize("mask", MASKS)
@pytest.mark.parametrize("tile", [1, 2, 3, 5, 16, 17])
def test_online_recurrence_equals_two_pass(mask, tile):
    """The tiled online-softmax recurrence equals the two-pass definition
    for any tile size, divisor of Sk or not (brute force, tiny sizes)."""
    Sq, Sk, causal, wl, wr = mask
    rng = np.random.default_rng(4 + tile)
    B, H, D = 1, 2, 8
    q, k, v = 3 * _rand(rng, B, Sq, H, D), _rand(rng, B, Sk, H, D), _rand(rng, B, Sk, H, D)
    o1, l1 = attention_forward(q, k, v, 0.6, causal, wl, wr)
    o2, l2 = online_softmax_forward(q, k, v, 0.6, tile, causal, wl, wr)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(np.isinf(l1), np.isinf(l2))
    f = np.isfinite(l1)
    np.testing.assert_allclose(l1[f], l2[f], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mask", [(6, 6, 0, -1, -1), (6, 6, 1, -1, -1), (5, 8, 1, 2, -1),
                                  (8, 5, 1, -1, -1), (7, 7, 0, 1, 1)])
def test_backward_matches_central_differences(mask):
    """Analytic dQ, dK, dV against central finite differences of
    L = sum(O * dO) in float64."""
    Sq, Sk, causal, wl, wr = mask
    rng = np.random.default_rng(5)
    B, H, D, scale = 1, 2, 4, 0.7
    q, k, v = _rand(rng, B, Sq, H, D), _rand(rng, B, Sk, H, D), _rand(rng, B, Sk, H, D)
    do = _rand(rng, B, Sq, H, D)
    g = attention_backward(q, k, v, do, scale, causal, wl, wr)

    def loss(qq, kk, vv):
        o, _ = attention_forward(qq, kk, vv, scale, causal, wl, wr)
        return float(np.sum(o * do))

    eps = 1e-5
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        num = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            args_p = [q, k, v]; args_m = [q, k, v]
            pos = {"dq": 0, "dk": 1, "dv": 2}[name]
            args_p[pos] = xp; args_m[pos] = xm
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        err = np.max(np.abs(num - g[name])) / max(1e-30, np.max(np.abs(num)))
        assert err < 1e-6, (name, err)


def test_window_zero_zero_copies_the_aligned_value_row():
    """win_left = win_right = 0: each query sees exactly key i + (Sk - Sq):
    O_i = V_{i+d}, LSE_i = scale * q_i . k_{i+d}."""
    rng = np.random.default_rng(6)
    B, Sq, Sk, H, D, scale = 2, 5, 8, 3, 4, 0.9
    q, k, v = _rand(rng, B, Sq, H, D), _rand(rng, B, Sk, H, D), _rand(rng, B, Sk, H, D)
    o, lse = attention_forward(q, k, v, scale, 0, 0, 0)
    d = Sk - Sq
    for b in range(B):
        for h in range(H):
            for i in range(Sq):
                np.testing.assert_allclose(o[b, i, h], v[b, i + d, h], rtol=1e-14, atol=1e-15)
                s = scale * sum(q[b, i, h, t] * k[b, i + d, h, t] for t in range(D))
                assert abs(lse[b, h, i] - s) < 1e-13


def test_single_key_returns_that_value():
    rng = np.random.default_rng(7)
    q, k, v = _rand(rng, 1, 6, 2, 3), _rand(rng, 1, 1, 2, 3), _rand(rng, 1, 1, 2, 3)
    o, lse = attention_forward(q, k, v, 1.3)
    for i in range(6):
        np.testing.assert_allclose(o[0, i], v[0, 0], rtol=1e-14)


def test_wide_window_equals_no_window():
    rng = np.random.default_rng(8)
    q, k, v = _rand(rng, 1, 12, 2, 4), _rand(rng, 1, 12, 2, 4), _rand(rng, 1, 12, 2, 4)
    for causal in (0, 1):
        a = attention_forward(q, k, v, 0.5, causal, -1, -1)
        b = attention_forward(q, k, v, 0.5, causal, 100, 100)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_window_rows_inside_the_window_equal_full_causal():
    """With window (W, 0) and causal, rows i <= W see every earlier key, so they
    equal the full-causal rows; later rows differ."""
    rng = np.random.default_rng(9)
    W = 5
    q, k, v = _rand(rng, 1, 16, 2, 4), _rand(rng, 1, 16, 2, 4), _rand(rng, 1, 16, 2, 4)
    ow, lw = attention_forward(q, k, v, 0.5, 1, W, 0)
    oc, lc = attention_forward(q, k, v, 0.5, 1, -1, -1)
    np.testing.assert_array_equal(ow[:, :W + 1], oc[:, :W + 1])
    assert np.max(np.abs(ow[:, W + 1:] - oc[:, W + 1:])) > 1e-3


def test_gradient_invariants():
    """Rows of P sum to one, so sum_j dV_j = sum_i dO_i (non-causal); the softmax
    is invariant to adding a common vector to all keys, so sum_j dK_j = 0; and
    with identical keys the scores are constant per row, so dQ = 0."""
    rng = np.random.default_rng(10)
    B, Sq, Sk, H, D = 1, 7, 9, 2, 5
    q, k, v, do = (_rand(rng, B, Sq, H, D), _rand(rng, B, Sk, H, D),
                   _rand(rng, B, Sk, H, D), _rand(rng, B, Sq, H, D))
    g = attention_backward(q, k, v, do, 0.8)
    np.testing.assert_allclose(g["dv"].sum(axis=1), do.sum(axis=1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g["dk"].sum(axis=1), 0.0, atol=1e-12)
    gc = attention_backward(q, k, v, do, 0.8, 1)   # causal: every row has a visible key
    np.testing.assert_allclose(gc["dk"].sum(axis=1), 0.0, atol=1e-12)
    np.testing.assert_allclose(gc["delta"], np.einsum("bshd,bshd->bhs", do, gc["o"]), rtol=1e-12, atol=1e-12)
    kc = np.repeat(k[:, :1], Sk, axis=1)
    g0 = attention_backward(q, kc, v, do, 0.8)
    np.testing.assert_allclose(g0["dq"], 0.0, atol=1e-12)


def test_row_and_head_helpers_agree_with_full_evaluation():
    rng = np.random.default_rng(11)
    B, Sq, Sk, H, D = 2, 10, 12, 3, 4
    q, k, v, do = (_rand(rng, B, Sq, H, D), _rand(rng, B, Sk, H, D),
                   _rand(rng, B, Sk, H, D), _rand(rng, B, Sq, H, D))
    for mask in [(1, -1, -1), (1, 3, 0), (0, -1, -1)]:
        g = attention_backward(q, k, v, do, 0.6, *mask)
        trip = np.array([[b, h, i] for b in range(B) for h in range(H) for i in range(Sq)])
        o_r, l_r = attention_forward_rows(q, k, v, trip, 0.6, *mask)
        dq_r, de_r = attention_backward_rows_dq(q, k, v, do, trip, 0.6, *mask)
        for t, (b, h, i) in enumerate(trip):
            np.testing.assert_allclose(o_r[t], g["o"][b, i, h], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(dq_r[t], g["dq"][b, i, h], rtol=1e-12, atol=1e-13)
            assert abs(l_r[t] - g["lse"][b, h, i]) < 1e-12
            assert abs(de_r[t] - g["delta"][b, h, i]) < 1e-12
        dk, dv = attention_backward_head(q, k, v, do, 1, 2, 0.6, *mask, row_chunk=3)
        np.testing.assert_allclose(dk, g["dk"][1, :, 2], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(dv, g["dv"][1, :, 2], rtol=1e-12, atol=1e-13)


def test_large_scores_do_not_overflow():
    """Scores near 700 would overflow exp without the max subtraction."""
    rng = np.random.default_rng(12)
    q = 100 * _rand(rng, 1, 8, 1, 4)
    k = 100 * _rand(rng, 1, 8, 1, 4)
    v = _rand(rng, 1, 8, 1, 4)
    o, lse = attention_forward(q, k, v, 1.0, 1)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    o2, l2 = online_softmax_forward(q, k, v, 1.0, 3, 1)
    np.testing.assert_allclose(o, o2, rtol=1e-10, atol=1e-12)
