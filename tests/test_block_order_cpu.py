"""Host-side checks of the index arithmetic the kernels choose their work with,
run on the CPU through the test-only diagnostics library (the functions are
the kernels' own host-and-device code; nothing is launched).

- mask bounds per query row and per key against the oracle's visibility
  matrix (FlashAttention-2 overview (lshu.cn), section 4.2 problem 4 for the
  causal mask; flash-attn install guide (yfxerp.com), section 1 for the
  window), and the monotonicity that the kernels' whole-tile tests rely on;
- the key-tile range of each forward query tile and the query-tile range of
  each backward key tile: every visible pair inside, no tile at either end
  without one;
- the chunked block order: a permutation of the grid, tile-major inside each
  chunk, head-major for chunks of one;
- the head_dim 256 backward's blocks: every dK, dV and dQ tile exactly once.
"""
import ctypes
import itertools
import os

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
DIAG = os.path.join(ROOT, "exact_attention_156_b200", "libattn156_diag.so")

_ip = ctypes.POINTER(ctypes.c_int)


@pytest.fixture(scope="module")
def diag():
    lib = ctypes.CDLL(DIAG)
    i = ctypes.c_int
    lib.attn_diag_mask_bounds.argtypes = [i, i, i, i, i, _ip, _ip, _ip, _ip]
    lib.attn_diag_fwd_tile_ranges.argtypes = [i, i, i, i, i, i, _ip, _ip, _ip, _ip]
    lib.attn_diag_bwd_qtile_ranges.argtypes = [i, i, i, i, i, i, _ip, _ip, _ip, _ip]
    lib.attn_diag_chunked_order.argtypes = [i, i, i, _ip, _ip]
    lib.attn_diag_d256_work.argtypes = [i, i, i, _ip, _ip]
    return lib


def _buf(n):
    a = np.zeros(max(n, 1), dtype=np.int32)
    return a, a.ctypes.data_as(_ip)


def _mask_bounds(diag, Sq, Sk, causal, wl, wr):
    lo, plo = _buf(Sq)
    hi, phi = _buf(Sq)
    qmin, pqmin = _buf(Sk)
    qmax, pqmax = _buf(Sk)
    assert diag.attn_diag_mask_bounds(Sq, Sk, causal, wl, wr, plo, phi, pqmin, pqmax) == 0
    return lo[:Sq], hi[:Sq], qmin[:Sk], qmax[:Sk]


MASKS = [(c, wl, wr) for c in (0, 1) for wl in (-1, 0, 1, 3, 9) for wr in (-1, 0, 2, 7)]


@pytest.mark.parametrize("causal,wl,wr", MASKS)
def test_mask_bounds_equal_the_oracle_visibility(diag, causal, wl, wr):
    for Sq, Sk in itertools.product((1, 2, 3, 7, 16, 33), (1, 2, 5, 16, 31, 40)):
        lo, hi, qmin, qmax = _mask_bounds(diag, Sq, Sk, causal, wl, wr)
        want = oracle.visible_mask(Sq, Sk, causal, wl, wr)
        i = np.arange(Sq)[:, None]
        j = np.arange(Sk)[None, :]
        by_rows = (j >= lo[:, None]) & (j <= hi[:, None])
        assert np.array_equal(by_rows, want), (Sq, Sk)
        by_keys = (i >= qmin[None, :]) & (i <= qmax[None, :])
        assert np.array_equal(by_keys, want), (Sq, Sk)
        # Both bounds grow with the row (and with the key): a tile's smallest
        # upper and largest lower bound sit at its first and last row, which
        # is what the kernels' whole-tile (no mask needed) tests read.
        assert np.all(np.diff(lo) >= 0) and np.all(np.diff(hi) >= 0)
        assert np.all(np.diff(qmin) >= 0) and np.all(np.diff(qmax) >= 0)


def _tiles_with_pairs(vis, rows, bn, n_key_tiles):
    """Key tiles holding at least one visible pair of the given query rows."""
    sub = vis[rows]
    return [t for t in range(n_key_tiles) if sub[:, t * bn:(t + 1) * bn].any()]


SHAPES = [(1, 1), (128, 128), (129, 300), (300, 129), (512, 512), (700, 450), (257, 1000)]
RANGE_MASKS = [(0, -1, -1), (1, -1, -1), (1, 200, 0), (0, 100, 50), (0, 0, 0), (1, 3, -1),
               (0, -1, 130)]


@pytest.mark.parametrize("Sq,Sk", SHAPES)
@pytest.mark.parametrize("causal,wl,wr", RANGE_MASKS)
def test_forward_key_tile_ranges_cover_every_visible_pair(diag, Sq, Sk, causal, wl, wr):
    bm_, bn_ = ctypes.c_int(), ctypes.c_int()
    _, pp = _buf(1)
    diag.attn_diag_fwd_tile_ranges(1, 1, 0, -1, -1, 1, pp, pp, ctypes.byref(bm_),
                                   ctypes.byref(bn_))
    bm, bn = bm_.value, bn_.value
    n = -(-Sq // bm) + 1  # and one tile past the end, where a pair's second tile can lie
    jlo, plo = _buf(n)
    jhi, phi = _buf(n)
    assert diag.attn_diag_fwd_tile_ranges(Sq, Sk, causal, wl, wr, n, plo, phi,
                                          ctypes.byref(bm_), ctypes.byref(bn_)) == 0
    vis = oracle.visible_mask(Sq, Sk, causal, wl, wr)
    nk = -(-Sk // bn)
    for t in range(n):
        rows = np.arange(t * bm, min((t + 1) * bm, Sq))
        have = _tiles_with_pairs(vis, rows, bn, nk) if len(rows) else []
        if not have:
            assert jhi[t] <= jlo[t], (t, jlo[t], jhi[t])
            continue
        assert jlo[t] == have[0] and jhi[t] == have[-1] + 1, (t, have, jlo[t], jhi[t])


@pytest.mark.parametrize("Sq,Sk", SHAPES)
@pytest.mark.parametrize("causal,wl,wr", RANGE_MASKS)
def test_backward_query_tile_ranges_cover_every_visible_pair(diag, Sq, Sk, causal, wl, wr):
    bm_, bn_ = ctypes.c_int(), ctypes.c_int()
    _, pp = _buf(1)
    diag.attn_diag_bwd_qtile_ranges(1, 1, 0, -1, -1, 1, pp, pp, ctypes.byref(bm_),
                                    ctypes.byref(bn_))
    bm, bn = bm_.value, bn_.value
    n = -(-Sk // bn)
    qlo, plo = _buf(n)
    qhi, phi = _buf(n)
    assert diag.attn_diag_bwd_qtile_ranges(Sq, Sk, causal, wl, wr, n, plo, phi,
                                           ctypes.byref(bm_), ctypes.byref(bn_)) == 0
    visT = oracle.visible_mask(Sq, Sk, causal, wl, wr).T
    nq = -(-Sq // bm)
    for t in range(n):
        keys = np.arange(t * bn, min((t + 1) * bn, Sk))
        have = _tiles_with_pairs(visT, keys, bm, nq)
        if not have:
            assert qhi[t] <= qlo[t], (t, qlo[t], qhi[t])
            continue
        assert qlo[t] == have[0] and qhi[t] == have[-1] + 1, (t, have, qlo[t], qhi[t])


def _chunked(diag, n_tiles, n_hb, chunk):
    tile, pt = _buf(n_tiles * n_hb)
    hb, ph = _buf(n_tiles * n_hb)
    assert diag.attn_diag_chunked_order(n_tiles, n_hb, chunk, pt, ph) == 0
    return tile[:n_tiles * n_hb], hb[:n_tiles * n_hb]


def test_chunked_order_is_a_permutation_tile_major_inside_each_chunk(diag):
    for n_tiles, n_hb in itertools.product((1, 2, 3, 8, 33), (1, 2, 5, 16, 17, 32, 40)):
        for chunk in sorted({1, 2, 3, 4, 7, 8, 16, n_hb, n_hb + 3}):
            tile, hb = _chunked(diag, n_tiles, n_hb, chunk)
            seen = set(zip(tile.tolist(), hb.tolist()))
            assert len(seen) == n_tiles * n_hb, (n_tiles, n_hb, chunk)
            assert seen == set(itertools.product(range(n_tiles), range(n_hb)))
            # chunks in order; inside one, tile 0 of every member, then tile 1, ...
            c = hb // chunk
            assert np.all(np.diff(c) >= 0)
            for ci in np.unique(c):
                sel = c == ci
                t, h = tile[sel], hb[sel]
                size = len(np.unique(h))
                assert np.array_equal(t, np.repeat(np.arange(n_tiles), size))
                assert np.array_equal(h, np.tile(np.sort(np.unique(h)), n_tiles))
            lin = np.arange(n_tiles * n_hb)
            if chunk == 1:  # head-major: the plain (x fastest) grid order
                assert np.array_equal(hb * n_tiles + tile, lin)
            if chunk >= n_hb:  # tile-major over the whole grid
                assert np.array_equal(tile * n_hb + hb, lin)


@pytest.mark.parametrize("causal", [0, 1])
def test_d256_backward_blocks_name_every_gradient_tile_once(diag, causal):
    DK, DV, DQ = 0, 1, 2
    for n_k, n_q in itertools.product(range(0, 9), range(0, 9)):
        n = 2 * n_k + n_q
        mode, pm = _buf(n)
        tile, pt = _buf(n)
        assert diag.attn_diag_d256_work(n_k, n_q, causal, pm, pt) == 0
        mode, tile = mode[:n], tile[:n]
        got = sorted(zip(mode.tolist(), tile.tolist()))
        want = sorted([(DK, t) for t in range(n_k)] + [(DV, t) for t in range(n_k)] +
                      [(DQ, t) for t in range(n_q)])
        assert got == want, (n_k, n_q)
        # key tiles in rising order (the most queries first under a causal
        # mask), dQ tiles heaviest first: falling when causal
        for m in (DK, DV):
            assert np.all(np.diff(tile[mode == m]) > 0)
        dq = tile[mode == DQ]
        assert np.all(np.diff(dq) < 0) if causal else np.all(np.diff(dq) > 0)
        # the first 3 min(n_k, n_q) blocks come in (dK l, dV l, dQ) threes
        nmin = min(n_k, n_q)
        assert np.array_equal(mode[:3 * nmin], np.tile([DK, DV, DQ], nmin))
        assert np.array_equal(tile[0:3 * nmin:3], np.arange(nmin))
        assert np.array_equal(tile[1:3 * nmin:3], np.arange(nmin))


def test_diag_rejects_bad_arguments(diag):
    _, p = _buf(4)
    assert diag.attn_diag_mask_bounds(-1, 4, 0, -1, -1, p, p, p, p) == 1
    assert diag.attn_diag_chunked_order(2, 2, 0, p, p) == 1
    assert diag.attn_diag_d256_work(-1, 2, 0, p, p) == 1
