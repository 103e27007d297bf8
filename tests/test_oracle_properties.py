"""Property checks of the oracle over random small shapes and masks (CPU):
the tiled online-softmax recurrence of the pages, with a random tile size,
equals the definition; and a packed batch of equal-length sequences equals the
batched oracle, forward and backward.  Derandomized, so runs are repeatable."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import (attention_backward, attention_backward_varlen, attention_forward,
                    attention_forward_varlen, online_softmax_forward)

shapes = st.tuples(
    st.integers(1, 2),          # B
    st.integers(1, 9),          # Sq
    st.integers(1, 9),          # Sk
    st.sampled_from([(1, 1), (2, 1), (2, 2), (4, 2), (3, 3)]),  # (H, Hk)
    st.sampled_from([1, 3, 4]),  # D
    st.booleans(),              # causal
    st.integers(-1, 4),         # win_left
    st.integers(-1, 4),         # win_right
    st.integers(0, 2**31 - 1),  # seed
)


def _draw(B, Sq, Sk, H, Hk, D, seed):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, Sq, H, D)), rng.standard_normal((B, Sk, Hk, D)),
            rng.standard_normal((B, Sk, Hk, D)), rng.standard_normal((B, Sq, H, D)))


@settings(max_examples=60, derandomize=True, deadline=None)
@given(shapes, st.integers(1, 10))
def test_online_recurrence_equals_the_definition(shape, tile):
    B, Sq, Sk, (H, Hk), D, causal, wl, wr, seed = shape
    q, k, v, _ = _draw(B, Sq, Sk, H, Hk, D, seed)
    o, lse = attention_forward(q, k, v, 0.7, int(causal), wl, wr)
    o2, lse2 = online_softmax_forward(q, k, v, 0.7, tile, int(causal), wl, wr)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse2[fin], lse[fin], atol=1e-12)


@settings(max_examples=40, derandomize=True, deadline=None)
@given(shapes)
def test_equal_length_packed_batch_equals_batched(shape):
    B, Sq, Sk, (H, Hk), D, causal, wl, wr, seed = shape
    q, k, v, do = _draw(B, Sq, Sk, H, Hk, D, seed)
    cq = np.arange(B + 1) * Sq
    ck = np.arange(B + 1) * Sk
    pack = lambda x: x.reshape(-1, x.shape[2], x.shape[3])
    o, lse = attention_forward_varlen(pack(q), pack(k), pack(v), cq, ck, 0.6, int(causal),
                                      wl, wr)
    o2, lse2 = attention_forward(q, k, v, 0.6, int(causal), wl, wr)
    np.testing.assert_allclose(o, pack(o2), atol=1e-13)
    lse2p = lse2.transpose(1, 0, 2).reshape(H, -1)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse2p))
    g = attention_backward_varlen(pack(q), pack(k), pack(v), pack(do), cq, ck, 0.6,
                                  int(causal), wl, wr)
    g2 = attention_backward(q, k, v, do, 0.6, int(causal), wl, wr)
    for name in ("dq", "dk", "dv"):
        np.testing.assert_allclose(g[name], pack(g2[name]), atol=1e-12)
