"""Pins for the oracle's grouped K/V heads (GQA; MQA when there is one K/V
head).  Query head h reads K/V head h // (H / Hk), and a shared K/V head's
gradient is the sum over the query heads that read it.  Each check ties the
grouped evaluation to facts that do not depend on the grouping code: the
independently pinned one-head-per-query-head oracle with K and V repeated,
central finite differences, and single-K/V-head special cases."""
import numpy as np
import pytest

from oracle import (attention_backward, attention_backward_head, attention_backward_kv_head,
                    attention_backward_rows_dq, attention_forward, attention_forward_rows,
                    kv_head, online_softmax_forward)

CASES = [
    # (B, Sq, Sk, H, Hk, causal, win_left, win_right)
    (1, 7, 7, 4, 2, 1, -1, -1),
    (2, 5, 9, 6, 3, 1, -1, -1),
    (1, 9, 9, 4, 1, 0, -1, -1),   # multi-query
    (1, 11, 11, 6, 2, 1, 3, 0),   # sliding window
]


def _inputs(case, seed):
    B, Sq, Sk, H, Hk, _, _, _ = case
    rng = np.random.default_rng(seed)
    D = 4
    q = rng.standard_normal((B, Sq, H, D))
    k = rng.standard_normal((B, Sk, Hk, D))
    v = rng.standard_normal((B, Sk, Hk, D))
    do = rng.standard_normal((B, Sq, H, D))
    return q, k, v, do


def _repeat(x, G):
    # K/V head g serves query heads g*G .. g*G + G - 1
    return np.repeat(x, G, axis=2)


@pytest.mark.parametrize("case", CASES)
def test_grouped_heads_equal_repeated_keys_and_values(case):
    B, Sq, Sk, H, Hk, causal, wl, wr = case
    q, k, v, do = _inputs(case, 11)
    G = H // Hk
    o, lse = attention_forward(q, k, v, 0.6, causal, wl, wr)
    o_r, lse_r = attention_forward(q, _repeat(k, G), _repeat(v, G), 0.6, causal, wl, wr)
    np.testing.assert_allclose(o, o_r, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lse_r, rtol=0, atol=1e-13)
    g = attention_backward(q, k, v, do, 0.6, causal, wl, wr)
    g_r = attention_backward(q, _repeat(k, G), _repeat(v, G), do, 0.6, causal, wl, wr)
    np.testing.assert_allclose(g["dq"], g_r["dq"], rtol=0, atol=1e-12)
    for name in ("dk", "dv"):
        summed = g_r[name].reshape(B, Sk, Hk, G, -1).sum(axis=3)
        np.testing.assert_allclose(g[name], summed, rtol=0, atol=1e-12)


def test_grouped_gradient_matches_central_differences():
    case = (1, 6, 6, 4, 2, 1, -1, -1)
    q, k, v, do = _inputs(case, 12)
    scale = 0.8
    g = attention_backward(q, k, v, do, scale, 1)

    def loss(kk, vv):
        o, _ = attention_forward(q, kk, vv, scale, 1)
        return float(np.sum(o * do))

    eps = 1e-5
    for name, x in (("dk", k), ("dv", v)):
        num = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp = x.copy(); xp[idx] += eps
            xm = x.copy(); xm[idx] -= eps
            if name == "dk":
                num[idx] = (loss(xp, v) - loss(xm, v)) / (2 * eps)
            else:
                num[idx] = (loss(k, xp) - loss(k, xm)) / (2 * eps)
        err = np.max(np.abs(num - g[name])) / np.max(np.abs(num))
        assert err < 1e-6, (name, err)


def test_single_key_value_head_serves_every_query_head():
    case = (1, 5, 5, 3, 1, 1, -1, -1)
    q, k, v, _ = _inputs(case, 13)
    o, lse = attention_forward(q, k, v, 0.5, 1)
    for h in range(3):
        o1, l1 = attention_forward(q[:, :, h:h + 1], k, v, 0.5, 1)
        np.testing.assert_allclose(o[:, :, h], o1[:, :, 0], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[:, h], l1[:, 0], rtol=0, atol=1e-14)


def test_grouped_helpers_agree_with_full_evaluation():
    case = (2, 9, 9, 6, 2, 1, -1, -1)
    B, Sq, Sk, H, Hk, causal, wl, wr = case
    q, k, v, do = _inputs(case, 14)
    full = attention_backward(q, k, v, do, 0.7, causal)
    triples = np.array([(b, h, i) for b in range(B) for h in range(H) for i in (0, 4, 8)])
    o_r, lse_r = attention_forward_rows(q, k, v, triples, 0.7, causal)
    dq_r, _ = attention_backward_rows_dq(q, k, v, do, triples, 0.7, causal)
    for n, (b, h, i) in enumerate(triples):
        np.testing.assert_allclose(o_r[n], full["o"][b, i, h], atol=1e-13)
        np.testing.assert_allclose(lse_r[n], full["lse"][b, h, i], atol=1e-13)
        np.testing.assert_allclose(dq_r[n], full["dq"][b, i, h], atol=1e-13)
    for b in range(B):
        for g in range(Hk):
            dk, dv = attention_backward_kv_head(q, k, v, do, b, g, 0.7, causal, row_chunk=4)
            np.testing.assert_allclose(dk, full["dk"][b, :, g], atol=1e-12)
            np.testing.assert_allclose(dv, full["dv"][b, :, g], atol=1e-12)
        # one query head's share, as the per-head helper gives it
        dk0, _ = attention_backward_head(q, k, v, do, b, 0, 0.7, causal)
        rep = attention_backward(q[:, :, 0:1], k[:, :, 0:1], v[:, :, 0:1], do[:, :, 0:1], 0.7, causal)
        np.testing.assert_allclose(dk0, rep["dk"][b, :, 0], atol=1e-12)


def test_online_recurrence_with_grouped_heads():
    case = (1, 7, 10, 4, 2, 1, 4, -1)
    q, k, v, _ = _inputs(case, 15)
    o1, l1 = attention_forward(q, k, v, 0.9, 1, 4, -1)
    o2, l2 = online_softmax_forward(q, k, v, 0.9, 3, 1, 4, -1)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(l1, l2, atol=1e-12)


def test_head_counts_must_divide():
    assert kv_head(5, 8, 2) == 1 and kv_head(7, 8, 8) == 7 and kv_head(3, 4, 1) == 0
    with pytest.raises(ValueError):
        kv_head(0, 6, 4)
    q = np.zeros((1, 3, 6, 4))
    k = np.zeros((1, 3, 4, 4))
    with pytest.raises(ValueError):
        attention_forward(q, k, k, 0.5)
