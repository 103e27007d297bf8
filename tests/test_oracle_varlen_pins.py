"""Pins for the oracle's packed variable-length batches: sequences of different
lengths stored back to back, delimited by cu_seqlens, each attending only
within itself.  Checked against facts that do not depend on the varlen code:
equal-length sequences reproduce the (independently pinned) batched oracle,
sequences never influence one another, brute-force per-row softmax on a
ragged batch with empty sequences, central finite differences of the packed
gradient, and refusal of malformed boundaries."""
import numpy as np
import pytest

from oracle import (attention_backward, attention_backward_varlen, attention_forward,
                    attention_forward_varlen)


def _packed(lq, lk, H, Hk, D, seed):
    rng = np.random.default_rng(seed)
    tq, tk = sum(lq), sum(lk)
    cq = np.concatenate([[0], np.cumsum(lq)])
    ck = np.concatenate([[0], np.cumsum(lk)])
    return (rng.standard_normal((tq, H, D)), rng.standard_normal((tk, Hk, D)),
            rng.standard_normal((tk, Hk, D)), rng.standard_normal((tq, H, D)), cq, ck)


@pytest.mark.parametrize("causal,wl,wr,Sq,Sk,Hk", [
    (0, -1, -1, 5, 5, 2), (1, -1, -1, 6, 6, 1), (1, -1, -1, 4, 7, 2), (1, 2, 0, 7, 7, 2),
    (0, 1, 2, 6, 4, 2)])
def test_equal_lengths_reproduce_the_batched_oracle(causal, wl, wr, Sq, Sk, Hk):
    B, H, D = 3, 4, 4
    q, k, v, do, cq, ck = _packed([Sq] * B, [Sk] * B, H, Hk, D, 11)
    o, lse = attention_forward_varlen(q, k, v, cq, ck, 0.6, causal, wl, wr)
    qb, kb, vb, dob = (x.reshape(B, -1, x.shape[1], D) for x in (q, k, v, do))
    o2, lse2 = attention_forward(qb, kb, vb, 0.6, causal, wl, wr)
    np.testing.assert_allclose(o, o2.reshape(o.shape), atol=1e-14)
    # batched LSE is (B, H, Sq); packed LSE is (H, total_q) with rows b*Sq + i
    np.testing.assert_array_equal(np.isneginf(lse), np.isneginf(lse2.transpose(1, 0, 2).reshape(H, -1)))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse2.transpose(1, 0, 2).reshape(H, -1)[fin], atol=1e-14)
    g = attention_backward_varlen(q, k, v, do, cq, ck, 0.6, causal, wl, wr)
    g2 = attention_backward(qb, kb, vb, dob, 0.6, causal, wl, wr)
    for name in ("dq", "dk", "dv"):
        np.testing.assert_allclose(g[name], g2[name].reshape(g[name].shape), atol=1e-13)


def test_sequences_do_not_influence_one_another():
    lq, lk = [3, 0, 5, 2], [4, 2, 5, 0]
    q, k, v, do, cq, ck = _packed(lq, lk, 2, 1, 4, 12)
    o, lse = attention_forward_varlen(q, k, v, cq, ck, 0.5, 1)
    g = attention_backward_varlen(q, k, v, do, cq, ck, 0.5, 1)
    # replace everything of sequence 2 by other values: sequences 0, 1, 3 stay bit-identical
    q2, k2, v2, do2 = q.copy(), k.copy(), v.copy(), do.copy()
    q2[cq[2]:cq[3]] = 7.0
    k2[ck[2]:ck[3]] = -3.0
    v2[ck[2]:ck[3]] = 1e3
    do2[cq[2]:cq[3]] = 5.0
    o2, lse2 = attention_forward_varlen(q2, k2, v2, cq, ck, 0.5, 1)
    g2 = attention_backward_varlen(q2, k2, v2, do2, cq, ck, 0.5, 1)
    rows = np.r_[cq[0]:cq[2], cq[3]:cq[4]]
    keys = np.r_[ck[0]:ck[2], ck[3]:ck[4]]
    np.testing.assert_array_equal(o[rows], o2[rows])
    np.testing.assert_array_equal(lse[:, rows], lse2[:, rows])
    np.testing.assert_array_equal(g["dq"][rows], g2["dq"][rows])
    np.testing.assert_array_equal(g["dk"][keys], g2["dk"][keys])
    np.testing.assert_array_equal(g["dv"][keys], g2["dv"][keys])


def test_brute_force_rows_of_a_ragged_batch():
    # lengths chosen so that some causal rows see no key (Lk < Lq) and one
    # sequence has no keys at all
    lq, lk = [4, 3, 2, 5], [6, 1, 0, 5]
    H, Hk, D = 4, 2, 3
    q, k, v, _, cq, ck = _packed(lq, lk, H, Hk, D, 13)
    o, lse = attention_forward_varlen(q, k, v, cq, ck, 0.8, 1)
    for b in range(4):
        Lq, Lk = lq[b], lk[b]
        for i in range(Lq):
            for h in range(H):
                g = h // (H // Hk)
                vis = [j for j in range(Lk) if j <= i + Lk - Lq]
                row = cq[b] + i
                if not vis:
                    assert np.all(o[row, h] == 0) and lse[h, row] == -np.inf
                    continue
                s = [0.8 * float(np.dot(q[row, h], k[ck[b] + j, g])) for j in vis]
                m = max(s)
                w = [np.exp(x - m) for x in s]
                ref = sum(wj * v[ck[b] + j, g] for wj, j in zip(w, vis)) / sum(w)
                np.testing.assert_allclose(o[row, h], ref, atol=1e-13)
                assert abs(lse[h, row] - (m + np.log(sum(w)))) < 1e-13


def test_packed_gradient_matches_central_differences():
    lq, lk = [3, 2, 4], [2, 3, 4]
    q, k, v, do, cq, ck = _packed(lq, lk, 2, 1, 3, 14)
    g = attention_backward_varlen(q, k, v, do, cq, ck, 0.7, 1, 2, -1)

    def loss(q_, k_, v_):
        o, _ = attention_forward_varlen(q_, k_, v_, cq, ck, 0.7, 1, 2, -1)
        return float(np.sum(o * do))

    eps = 1e-6
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += eps
            xm[idx] -= eps
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * eps)
        np.testing.assert_allclose(g[name], num, atol=2e-7, rtol=1e-6)


def test_malformed_boundaries_are_refused():
    q, k, v, _, cq, ck = _packed([2, 3], [2, 3], 1, 1, 2, 15)
    for bad_q, bad_k in (([1, 2, 5], ck), ([0, 3, 2], ck), ([0, 2, 4], ck), (cq, [0, 2])):
        with pytest.raises(ValueError):
            attention_forward_varlen(q, k, v, bad_q, bad_k, 0.5, 0)
