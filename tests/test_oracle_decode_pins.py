"""Pins for the oracle's KV-cache decode: a few query rows per sequence against
the first cache_seqlens[b] rows of a cache.  Checked against facts that do not
depend on the decode code: full-length caches equal ordinary attention (itself
pinned), cache rows past the length are never read, a one-key cache returns
that value row, causal decode rows equal the last rows of a full causal
attention, and brute-force per-row softmax."""
import numpy as np
import pytest

from oracle import attention_decode, attention_forward


def _inputs(B, Sq, Smax, H, Hk, D, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Sq, H, D)), rng.standard_normal((B, Smax, Hk, D)),
            rng.standard_normal((B, Smax, Hk, D)))


def test_full_caches_equal_ordinary_attention():
    q, k, v = _inputs(2, 3, 9, 4, 2, 8, 1)
    for causal in (0, 1):
        o, lse = attention_decode(q, k, v, [9, 9], 0.4, causal)
        o2, lse2 = attention_forward(q, k, v, 0.4, causal)
        np.testing.assert_allclose(o, o2, atol=1e-14)
        np.testing.assert_allclose(lse, lse2, atol=1e-14)


def test_rows_past_the_length_are_never_read():
    q, k, v = _inputs(3, 2, 12, 2, 1, 8, 2)
    lens = [5, 12, 1]
    o, lse = attention_decode(q, k, v, lens, 0.5, 1)
    k2, v2 = k.copy(), v.copy()
    for b, L in enumerate(lens):
        k2[b, L:] = 1e6
        v2[b, L:] = np.nan
    o2, lse2 = attention_decode(q, k2, v2, lens, 0.5, 1)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


def test_single_cached_key_returns_its_value():
    q, k, v = _inputs(1, 1, 6, 3, 3, 4, 3)
    o, lse = attention_decode(q, k, v, [1], 0.7, 0)
    for h in range(3):
        np.testing.assert_allclose(o[0, 0, h], v[0, 0, h], atol=1e-15)
        np.testing.assert_allclose(lse[0, h, 0], 0.7 * q[0, 0, h] @ k[0, 0, h], atol=1e-14)


def test_causal_decode_rows_are_the_last_rows_of_full_attention():
    rng = np.random.default_rng(4)
    L, Sq = 11, 3
    q_all = rng.standard_normal((1, L, 2, 8))
    k = rng.standard_normal((1, 16, 2, 8))
    v = rng.standard_normal((1, 16, 2, 8))
    o_full, lse_full = attention_forward(q_all, k[:, :L], v[:, :L], 0.3, 1)
    o, lse = attention_decode(q_all[:, L - Sq:], k, v, [L], 0.3, 1)
    np.testing.assert_allclose(o[0], o_full[0, L - Sq:], atol=1e-14)
    np.testing.assert_allclose(lse[0], lse_full[0, :, L - Sq:], atol=1e-14)


def test_brute_force_rows():
    q, k, v = _inputs(2, 2, 7, 4, 2, 4, 5)
    lens = [4, 7]
    o, lse = attention_decode(q, k, v, lens, 0.9, 1)
    for b, L in enumerate(lens):
        for h in range(4):
            g = h // 2
            for i in range(2):
                n = L - 2 + i + 1  # visible keys 0 .. L-2+i
                s = [0.9 * float(np.dot(q[b, i, h], k[b, j, g])) for j in range(n)]
                m = max(s)
                w = [np.exp(x - m) for x in s]
                z = sum(w)
                ref = sum(w[j] * v[b, j, g] for j in range(n)) / z
                np.testing.assert_allclose(o[b, i, h], ref, atol=1e-13)
                assert abs(lse[b, h, i] - (m + np.log(z))) < 1e-13


def test_empty_cache_gives_rows_with_no_visible_key():
    """A zero-length cache leaves every row of that sequence without a visible
    key: O = 0 and LSE = -inf (the rule for such rows everywhere), and the other
    sequences are unaffected."""
    q, k, v = _inputs(2, 2, 4, 1, 1, 4, 6)
    o, lse = attention_decode(q, k, v, [0, 3], 0.5, 0)
    assert np.all(o[0] == 0) and np.all(np.isneginf(lse[0]))
    o1, lse1 = attention_decode(q[1:], k[1:], v[1:], [3], 0.5, 0)
    np.testing.assert_array_equal(o[1], o1[0])
    np.testing.assert_array_equal(lse[1], lse1[0])
    with pytest.raises(ValueError):
        attention_decode(q, k, v, [-1, 3], 0.5, 0)
