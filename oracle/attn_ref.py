"""Float64 CPU oracle for exact scaled dot-product attention and its gradient.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It shares no code with the CUDA path.

What it computes.  The pages call the method exact (FlashAttention-2
overview, lshu.cn, section 1; flash-attn install guide, yfxerp.com,
section 1, which describes it as exact and IO-aware), so the oracle is
the plain definition, the standard attention of the FlashAttention-2 overview,
section 2.1 (first anti-pattern): scores S = Q K^T, a row-wise softmax with
the row maximum subtracted first (section 2.1, third anti-pattern, on
stability), then the weighted sum of V.  Everything runs in float64 on the
given (already bf16-rounded) inputs; no tiling, fusion or reordering.

Readings of points the pages leave open:
  * scale multiplies the scores: S = scale * Q K^T.  ``softmax_scale=None``
    in the pages' ``flash_attn_func`` call (section 3.3 snippet) means
    1/sqrt(head_dim); callers here always pass it explicitly.
  * causal (an upper-triangular mask, section 4.2 problem 4) is aligned to the
    bottom-right corner: key j is visible to query i iff j <= i + (Sk - Sq).
  * window (``window_size`` is only named on the yfxerp.com page, section 1):
    with delta = Sk - Sq, key j is visible to query i iff
    (win_left < 0 or j >= i + delta - win_left) and
    (win_right < 0 or j <= i + delta + win_right), and with the causal rule
    when causal is set.  Both bounds are inclusive.
  * LSE (not on the pages) is the natural log-sum-exp of the scaled, masked
    scores: LSE_i = m_i + ln(sum_j exp(S_ij - m_i)).
  * a query row with no visible key has O_i = 0, LSE_i = -inf and zero
    gradient contributions.
  * K and V may have fewer heads Hk than Q (H a multiple of Hk): the pages'
    Transformers snippet (FlashAttention-2 overview, lshu.cn, section 3.3)
    shapes Q with num_heads and K, V with num_kv_heads for the same call.
    Query head h attends with key/value head h // (H / Hk) (consecutive query
    heads share one K/V head; Hk = 1 is multi-query attention), and the
    gradient of a shared K/V head is the sum over its query heads.
  * the backward is the analytic gradient of that definition (the pages say
    only that the backward recomputes the scores, yfxerp.com section 1):
    dV = P^T dO; dP = dO V^T; Delta_i = sum_j P_ij dP_ij; dS = P * (dP - Delta);
    dQ = scale * dS K; dK = scale * dS^T Q.

Arrays use the pages' layout (batch, seqlen, nheads, head_dim).
"""
from __future__ import annotations

import numpy as np


def kv_head(h: int, H: int, Hk: int) -> int:
    """Key/value head used by query head h when K and V have Hk of H heads."""
    if Hk < 1 or H % Hk != 0:
        raise ValueError(f"query heads {H} not a multiple of key/value heads {Hk}")
    return h // (H // Hk)


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def visible_mask(Sq: int, Sk: int, causal: int, win_left: int = -1,
                 win_right: int = -1, rows=None) -> np.ndarray:
    """Boolean (Sq, Sk) matrix: True where key j is visible to query i (only
    the given query rows, in that order, when ``rows`` is given).

    Causal mask: FlashAttention-2 overview (lshu.cn), section 4.2 problem 4
    (upper-triangular mask, each token sees only earlier tokens); window:
    flash-attn install guide (yfxerp.com), section 1 (``window_size``).
    Alignment and inclusive bounds are this oracle's stated reading.
    """
    i = (np.arange(Sq, dtype=np.int64) if rows is None
         else np.asarray(rows, dtype=np.int64))[:, None]
    j = np.arange(Sk, dtype=np.int64)[None, :]
    delta = Sk - Sq
    vis = np.ones((i.shape[0], Sk), dtype=bool)
    if causal:
        vis &= j <= i + delta
    if win_left >= 0:
        vis &= j >= i + delta - win_left
    if win_right >= 0:
        vis &= j <= i + delta + win_right
    return vis


def _softmax_rows(S: np.ndarray):
    """Stable row softmax of a masked score block (rows x keys, -inf = masked).

    Returns (P, lse): the row maximum is subtracted before exponentiating
    (FlashAttention-2 overview, section 2.1, third anti-pattern).  Rows with no
    visible key get P = 0 and lse = -inf.
    """
    m = np.max(S, axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    m_safe = np.where(empty, 0.0, m)
    E = np.exp(S - m_safe)  # exp(-inf) = 0 for masked entries
    l = np.sum(E, axis=-1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        P = np.where(empty, 0.0, E / np.where(empty, 1.0, l))
        lse = np.where(empty, -np.inf, m_safe + np.log(np.where(empty, 1.0, l)))
    return P, lse[..., 0]


def _scores(qh, kh, scale, rows, Sq, Sk, causal, wl, wr):
    """scale * Q K^T for the given query rows of one head, masked with -inf."""
    S = scale * (qh @ kh.T)
    vis = visible_mask(Sq, Sk, causal, wl, wr, rows=rows)
    return np.where(vis, S, -np.inf)


def attention_forward(q, k, v, scale: float, causal: int = 0,
                      win_left: int = -1, win_right: int = -1):
    """O and LSE of exact attention, the three standard steps in float64.

    q: (B, Sq, H, D); k, v: (B, Sk, Hk, D) with H a multiple of Hk.  Returns
    o (B, Sq, H, D) float64 and lse (B, H, Sq) float64 (natural log).
    FlashAttention-2 overview (lshu.cn), section 2.1: S = Q K^T, row softmax,
    weighted sum of V.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    o = np.zeros((B, Sq, H, D), dtype=np.float64)
    lse = np.zeros((B, H, Sq), dtype=np.float64)
    rows = np.arange(Sq)
    Hk = k.shape[2]
    for b in range(B):
        for h in range(H):
            g = kv_head(h, H, Hk)
            S = _scores(q[b, :, h, :], k[b, :, g, :], scale, rows, Sq, Sk,
                        causal, win_left, win_right)
            P, l = _softmax_rows(S)
            o[b, :, h, :] = P @ v[b, :, g, :]
            lse[b, h, :] = l
    return o, lse


def attention_forward_rows(q, k, v, triples, scale: float, causal: int = 0,
                           win_left: int = -1, win_right: int = -1):
    """O and LSE for selected (batch, head, row) triples only.

    Each output row depends only on its own query row and all keys of its
    (batch, head), so the definition is evaluated row by row in float64.
    Returns (o_rows (m, D), lse_rows (m,)) in the order of ``triples``.
    """
    q, k, v = np.asarray(q), np.asarray(k), np.asarray(v)
    triples = np.asarray(triples, dtype=np.int64)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    o = np.zeros((len(triples), D), dtype=np.float64)
    lse = np.zeros((len(triples),), dtype=np.float64)
    # group by (b, h) so K and V of a head are widened once
    keys = triples[:, 0] * H + triples[:, 1]
    for bh in np.unique(keys):
        sel = np.nonzero(keys == bh)[0]
        b, h = int(bh // H), int(bh % H)
        g = kv_head(h, H, k.shape[2])
        kh = _f64(k[b, :, g, :])
        vh = _f64(v[b, :, g, :])
        for c0 in range(0, len(sel), 1024):
            s = sel[c0:c0 + 1024]
            rows = triples[s, 2]
            qh = _f64(q[b, rows, h, :])
            S = _scores(qh, kh, scale, rows, Sq, Sk, causal, win_left, win_right)
            P, l = _softmax_rows(S)
            o[s] = P @ vh
            lse[s] = l
    return o, lse


def _head_backward(qh, kh, vh, doh, scale, rows, Sq, Sk, causal, wl, wr):
    """Analytic gradient pieces for a block of query rows of one head."""
    S = _scores(qh, kh, scale, rows, Sq, Sk, causal, wl, wr)
    P, lse = _softmax_rows(S)
    O = P @ vh
    dP = doh @ vh.T
    delta = np.sum(P * dP, axis=-1, keepdims=True)
    dS = P * (dP - delta)
    return O, lse, delta[:, 0], P, dS


def attention_backward(q, k, v, do, scale: float, causal: int = 0,
                       win_left: int = -1, win_right: int = -1):
    """Analytic gradient of L = sum(O * dO) with respect to Q, K and V.

    Returns a dict with o, lse, delta (B, H, Sq), dq, dk, dv (float64); with
    fewer K/V heads, dk and dv of a K/V head sum over its query heads.
    dV = P^T dO; dP = dO V^T; Delta = rowsum(P * dP) (= rowsum(dO * O));
    dS = P * (dP - Delta); dQ = scale dS K; dK = scale dS^T Q.
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    out = {name: np.zeros_like(x) for name, x in
           (("o", q), ("dq", q), ("dk", k), ("dv", v))}
    out["lse"] = np.zeros((B, H, Sq))
    out["delta"] = np.zeros((B, H, Sq))
    rows = np.arange(Sq)
    Hk = k.shape[2]
    for b in range(B):
        for h in range(H):
            g = kv_head(h, H, Hk)
            qh, kh, vh, doh = q[b, :, h], k[b, :, g], v[b, :, g], do[b, :, h]
            O, lse, delta, P, dS = _head_backward(qh, kh, vh, doh, scale, rows,
                                                  Sq, Sk, causal, win_left, win_right)
            out["o"][b, :, h] = O
            out["lse"][b, h] = lse
            out["delta"][b, h] = delta
            out["dv"][b, :, g] += P.T @ doh
            out["dq"][b, :, h] = scale * (dS @ kh)
            out["dk"][b, :, g] += scale * (dS.T @ qh)
    return out


def attention_backward_rows_dq(q, k, v, do, triples, scale: float, causal: int = 0,
                               win_left: int = -1, win_right: int = -1):
    """dQ for selected (batch, head, row) triples; each dQ row is row-local.

    Returns (dq_rows (m, D), delta_rows (m,)).
    """
    q, k, v, do = np.asarray(q), np.asarray(k), np.asarray(v), np.asarray(do)
    triples = np.asarray(triples, dtype=np.int64)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    dq = np.zeros((len(triples), D))
    dl = np.zeros((len(triples),))
    keys = triples[:, 0] * H + triples[:, 1]
    for bh in np.unique(keys):
        sel = np.nonzero(keys == bh)[0]
        b, h = int(bh // H), int(bh % H)
        g = kv_head(h, H, k.shape[2])
        kh, vh = _f64(k[b, :, g]), _f64(v[b, :, g])
        for c0 in range(0, len(sel), 1024):
            s = sel[c0:c0 + 1024]
            rows = triples[s, 2]
            _, _, delta, _, dS = _head_backward(_f64(q[b, rows, h]), kh, vh,
                                                _f64(do[b, rows, h]), scale, rows,
                                                Sq, Sk, causal, win_left, win_right)
            dq[s] = scale * (dS @ kh)
            dl[s] = delta
    return dq, dl


def attention_backward_rows(q, k, v, do, b: int, h: int, rows, scale: float,
                            causal: int = 0, win_left: int = -1, win_right: int = -1):
    """Forward and backward pieces owed to a set of query rows of one head.

    Returns (o_rows, lse_rows, dq_rows, dk_part, dv_part): O, LSE and dQ of
    the given rows, and the terms those rows add to dK and dV (sum over rows
    of dS^T Q and P^T dO).  Summing dk_part/dv_part over a partition of the
    rows gives the head's dK and dV.
    """
    rows = np.asarray(rows, dtype=np.int64)
    Sq = q.shape[1]
    Sk = k.shape[1]
    g = kv_head(h, q.shape[2], k.shape[2])
    kh, vh = _f64(k[b, :, g]), _f64(v[b, :, g])
    qh, doh = _f64(q[b, rows, h]), _f64(do[b, rows, h])
    O, lse, _, P, dS = _head_backward(qh, kh, vh, doh, scale, rows, Sq, Sk,
                                      causal, win_left, win_right)
    return O, lse, scale * (dS @ kh), scale * (dS.T @ qh), P.T @ doh


def attention_backward_head(q, k, v, do, b: int, h: int, scale: float,
                            causal: int = 0, win_left: int = -1, win_right: int = -1,
                            row_chunk: int = 1024):
    """Query head h's share of dK and dV (Sk, D) of its (batch, K/V head);
    query rows are taken in chunks.  With as many K/V heads as query heads
    this is the head's dK and dV.

    dK and dV sum over every query row, so every row's softmax and Delta is
    evaluated; chunking the rows only bounds memory.
    """
    Sq = q.shape[1]
    Sk = k.shape[1]
    D = k.shape[3]
    dk = np.zeros((Sk, D))
    dv = np.zeros((Sk, D))
    for r0 in range(0, Sq, row_chunk):
        rows = np.arange(r0, min(Sq, r0 + row_chunk))
        _, _, _, dkp, dvp = attention_backward_rows(q, k, v, do, b, h, rows, scale,
                                                    causal, win_left, win_right)
        dk += dkp
        dv += dvp
    return dk, dv


def attention_backward_kv_head(q, k, v, do, b: int, g: int, scale: float,
                               causal: int = 0, win_left: int = -1, win_right: int = -1,
                               row_chunk: int = 1024):
    """dK and dV (Sk, D) of K/V head g of batch b: the sum over the query
    heads that share it (just one when the head counts are equal)."""
    H, Hk = q.shape[2], k.shape[2]
    dk = np.zeros((k.shape[1], k.shape[3]))
    dv = np.zeros_like(dk)
    for h in range(H):
        if kv_head(h, H, Hk) == g:
            dkh, dvh = attention_backward_head(q, k, v, do, b, h, scale, causal,
                                               win_left, win_right, row_chunk)
            dk += dkh
            dv += dvh
    return dk, dv


def attention_decode(q, k_cache, v_cache, cache_seqlens, scale: float, causal: int = 0):
    """O and LSE for a few new query rows per sequence against a K/V cache.

    FlashAttention-2 overview (lshu.cn), section 3.3: flash_attn_func has no
    incremental (KV-cache) path and flash_attn_with_kvcache is the entry point
    for it; the pages give no further semantics.  Reading: q (B, Sq, H, D) holds
    the Sq newest query rows of each sequence, k_cache, v_cache (B, Smax, Hk, D)
    hold that sequence's keys and values in their first cache_seqlens[b] rows
    (the new keys already appended), and those rows are all the keys it
    attends over; rows past the length are never read.  Causal is the same
    bottom-right rule as everywhere (query i of Sq sees keys
    j <= i + cache_seqlens[b] - Sq).  Returns o (B, Sq, H, D), lse (B, H, Sq).
    """
    q = _f64(q)
    B, Sq, H, D = q.shape
    o = np.zeros((B, Sq, H, D))
    lse = np.zeros((B, H, Sq))
    for b in range(B):
        L = int(cache_seqlens[b])
        if L < 0:
            raise ValueError("cache lengths are counts of rows")
        if L == 0:
            # no key to attend to: every row of the sequence is a row with no
            # visible key, O = 0 and LSE = -inf as in attention_forward
            lse[b] = -np.inf
            continue
        ob, lb = attention_forward(q[b:b + 1], _f64(k_cache[b:b + 1, :L]),
                                   _f64(v_cache[b:b + 1, :L]), scale, causal)
        o[b] = ob[0]
        lse[b] = lb[0]
    return o, lse


def _cu_seqlens(cu, total: int, name: str):
    """Sequence boundaries: cu[0] = 0, non-decreasing, cu[-1] = total."""
    cu = np.asarray(cu, dtype=np.int64)
    if cu.ndim != 1 or cu.size < 2 or cu[0] != 0 or cu[-1] != total or np.any(np.diff(cu) < 0):
        raise ValueError(f"{name} must start at 0, never decrease and end at {total}")
    return cu


def attention_forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float,
                             causal: int = 0, win_left: int = -1, win_right: int = -1):
    """O and LSE for a batch of sequences of different lengths packed end to end.

    The pages only name the upstream tests for variable-length and padded
    batches (FlashAttention-2 overview, lshu.cn, section 3.2).  Reading:
    q (total_q, H, D) and k, v (total_k, Hk, D) hold the sequences back to
    back; sequence b is rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 of q and
    cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1 of k and v, and attends only within
    itself, with the masks applied to its own lengths (bottom-right causal per
    sequence).  A sequence with no keys gives its rows O = 0, LSE = -inf.
    Returns o (total_q, H, D) and lse (H, total_q).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    cq = _cu_seqlens(cu_seqlens_q, q.shape[0], "cu_seqlens_q")
    ck = _cu_seqlens(cu_seqlens_k, k.shape[0], "cu_seqlens_k")
    if cq.size != ck.size:
        raise ValueError("cu_seqlens_q and cu_seqlens_k describe different batch sizes")
    H = q.shape[1]
    o = np.zeros_like(q)
    lse = np.full((H, q.shape[0]), -np.inf)
    for b in range(cq.size - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue  # no rows, or rows that see no key (O = 0, LSE = -inf)
        ob, lb = attention_forward(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], scale,
                                   causal, win_left, win_right)
        o[q0:q1] = ob[0]
        lse[:, q0:q1] = lb[0]
    return o, lse


def attention_backward_varlen(q, k, v, do, cu_seqlens_q, cu_seqlens_k, scale: float,
                              causal: int = 0, win_left: int = -1, win_right: int = -1):
    """Gradient of L = sum(O * dO) for packed variable-length sequences (the
    layout and reading of ``attention_forward_varlen``).  Each sequence's
    gradient is that of its own attention; sequences never mix.  Returns a dict
    with o, dq (total_q, H, D), dk, dv (total_k, Hk, D), lse, delta (H, total_q).
    """
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    cq = _cu_seqlens(cu_seqlens_q, q.shape[0], "cu_seqlens_q")
    ck = _cu_seqlens(cu_seqlens_k, k.shape[0], "cu_seqlens_k")
    if cq.size != ck.size:
        raise ValueError("cu_seqlens_q and cu_seqlens_k describe different batch sizes")
    H = q.shape[1]
    out = {"o": np.zeros_like(q), "dq": np.zeros_like(q), "dk": np.zeros_like(k),
           "dv": np.zeros_like(v), "lse": np.full((H, q.shape[0]), -np.inf),
           "delta": np.zeros((H, q.shape[0]))}
    for b in range(cq.size - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0 or k1 == k0:
            continue  # nothing visible: zero output and zero gradients
        r = attention_backward(q[None, q0:q1], k[None, k0:k1], v[None, k0:k1], do[None, q0:q1],
                               scale, causal, win_left, win_right)
        out["o"][q0:q1] = r["o"][0]
        out["dq"][q0:q1] = r["dq"][0]
        out["dk"][k0:k1] = r["dk"][0]
        out["dv"][k0:k1] = r["dv"][0]
        out["lse"][:, q0:q1] = r["lse"][0]
        out["delta"][:, q0:q1] = r["delta"][0]
    return out


def online_softmax_forward(q, k, v, scale: float, tile: int, causal: int = 0,
                           win_left: int = -1, win_right: int = -1):
    """The pages' online-softmax recurrence, one key tile at a time.

    FlashAttention-2 overview (lshu.cn), section 2.2, innovation 2: keep a
    running row maximum m_i and running sum l_i = sum_j exp(qk_j - m_i),
    updated as each tile of scores is produced, so the full score row is
    never stored; section 2.2 innovation 1 gives the tile loop (load a Q
    block, then for each K/V block: local Q K^T, local softmax, weighted sum
    of the V block).  The accumulator is kept unnormalised and divided by
    l_i once at the end (equal in exact arithmetic to normalising per tile).
    Used only to pin the definition in ``attention_forward`` (they must agree
    to rounding); ``tile`` may be any positive size, divisor or not.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Sq, H, D = q.shape
    Sk = k.shape[1]
    vis = visible_mask(Sq, Sk, causal, win_left, win_right)
    o = np.zeros((B, Sq, H, D))
    lse = np.zeros((B, H, Sq))
    for b in range(B):
        for h in range(H):
            g = kv_head(h, H, k.shape[2])
            for i in range(Sq):
                m_i = -np.inf
                l_i = 0.0
                acc = np.zeros(D)
                for j0 in range(0, Sk, tile):
                    j1 = min(Sk, j0 + tile)
                    s = scale * (k[b, j0:j1, g] @ q[b, i, h])
                    s = np.where(vis[i, j0:j1], s, -np.inf)
                    m_new = max(m_i, float(np.max(s)))
                    if m_new == -np.inf:
                        continue  # nothing visible yet
                    alpha = np.exp(m_i - m_new)  # exp(-inf) = 0 on the first visible tile
                    p = np.exp(s - m_new)
                    l_i = l_i * alpha + float(np.sum(p))
                    acc = acc * alpha + p @ v[b, j0:j1, g]
                    m_i = m_new
                if l_i > 0.0:
                    o[b, i, h] = acc / l_i
                    lse[b, h, i] = m_i + np.log(l_i)
                else:
                    lse[b, h, i] = -np.inf
    return o, lse
