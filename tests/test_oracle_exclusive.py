"""Pins of the oracle's window-exclusive selection reading.

Reading (demingchina commentary on HySparse2, section 03): the sparse layers
see k "global" tokens plus the latest w, so the top-k draws only from blocks
that end before the forced window of the tile's last query. These CPU tests
tie that reading to plain-Python enumerations and to the method's invariants:
with w = 0 it is the union reading; the kept blocks are the top-k of the
restricted candidate list (score descending, lower index first) and never
reach into the last query's window; at one query per tile the selected and
window keys are disjoint, so |V_q| = k + w; with every candidate kept the
sparse layer is full attention; with no candidate it is the window alone.
Reading of "before the window" at block granularity: a block competes if its
first key precedes the window of the tile's last query.
"""
import math

import numpy as np
import pytest

import oracle as O

RNG = np.random.default_rng(23)


def _case(ctx, new, Hkv=1):
    kv = [c + n for c, n in zip(ctx, new)]
    cu_q = [0] + [int(x) for x in np.cumsum(new)]
    cu_kv = [0] + [int(x) for x in np.cumsum(kv)]
    return cu_q, cu_kv


def _level_scores(n_tiles, Hkv, nblk):
    # a few levels so that ties straddle the k-th place
    return RNG.choice([0.125, 0.25, 0.5, 1.0], size=(n_tiles, Hkv, nblk))


@pytest.mark.parametrize("T,B,k", [(4, 1, 5), (8, 2, 3), (1, 1, 7)])
def test_exclusive_with_no_window_is_the_union_reading(T, B, k):
    cu_q, cu_kv = _case((5, 0, 31), (13, 9, 6))
    nblk = (max(b - a for a, b in zip(cu_kv, cu_kv[1:])) + B - 1) // B
    sc = _level_scores(len(O.make_tiles(cu_q, cu_kv, T)), 2, nblk)
    a = O.topk_select(sc, cu_q, cu_kv, T, B, k)
    b = O.topk_select(sc, cu_q, cu_kv, T, B, k, w=0, exclusive=True)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


@pytest.mark.parametrize("T,B,w,k", [(4, 1, 3, 5), (8, 1, 6, 2), (5, 2, 4, 3), (1, 1, 4, 6), (3, 4, 5, 2)])
def test_exclusive_keeps_the_top_k_of_the_restricted_candidates(T, B, w, k):
    cu_q, cu_kv = _case((7, 0, 40), (14, 11, 9))
    tiles = O.make_tiles(cu_q, cu_kv, T)
    nblk = (max(b - a for a, b in zip(cu_kv, cu_kv[1:])) + B - 1) // B
    sc = _level_scores(len(tiles), 2, nblk)
    idx, cnt = O.topk_select(sc, cu_q, cu_kv, T, B, k, w=w, exclusive=True)
    for t in tiles:
        lim = t.last_pos - w  # candidate blocks start at or before lim
        cand = [b for b in range(nblk) if b * B <= lim]
        for g in range(2):
            # plain Python: sort candidates by (score descending, index ascending)
            order = sorted(cand, key=lambda b: (-sc[t.index, g, b], b))
            want = sorted(order[:k])
            got = idx[t.index, g, :cnt[t.index, g]].tolist()
            assert got == want
            assert cnt[t.index, g] == min(k, len(cand))
            assert (idx[t.index, g, cnt[t.index, g]:] == -1).all()
            # every kept block starts before the last query's window
            assert all(b * B <= lim for b in got)


def test_one_query_per_tile_sees_k_plus_w_distinct_keys():
    # decode shape: T = 1, token level; long enough that k candidates exist
    w, k = 5, 7
    cu_q, cu_kv = _case((30, 12, 3), (1, 1, 1))
    tiles = O.make_tiles(cu_q, cu_kv, 1)
    nblk = max(b - a for a, b in zip(cu_kv, cu_kv[1:]))
    sc = RNG.random((len(tiles), 1, nblk)) + 0.01
    idx, cnt = O.topk_select(sc, cu_q, cu_kv, 1, 1, k, w=w, exclusive=True)
    for t in tiles:
        vis = O.sparse_visible(t, idx[t.index, 0, :cnt[t.index, 0]], 1, w)
        pos = t.last_pos
        n_sel = min(k, max(0, pos - w + 1))
        n_win = min(w, pos + 1)
        assert int(vis[0].sum()) == n_sel + n_win
        # and the union reading, whose top-k may fall inside the window, sees fewer or as many
        iu, cu = O.topk_select(sc, cu_q, cu_kv, 1, 1, k)
        vu = O.sparse_visible(t, iu[t.index, 0, :cu[t.index, 0]], 1, w)
        assert int(vu[0].sum()) <= n_sel + n_win


def _rand_qkv(cu_q, cu_kv, Hq=4, Hkv=1, d=8):
    q = RNG.standard_normal((cu_q[-1], Hq, d))
    k = RNG.standard_normal((cu_kv[-1], Hkv, d))
    v = RNG.standard_normal((cu_kv[-1], Hkv, d))
    return q, k, v


@pytest.mark.parametrize("T,B,w", [(4, 1, 3), (6, 2, 4), (1, 1, 2)])
def test_exclusive_with_every_candidate_kept_is_full_attention(T, B, w):
    cu_q, cu_kv = _case((9, 0), (12, 10))
    q, k, v = _rand_qkv(cu_q, cu_kv)
    o_f, lse_f = O.full_attention(q, k, v, cu_q, cu_kv, 1)
    _, lse_t = O.full_attention(q, k, v, cu_q, cu_kv, 1, tiles_T=T)
    sc = O.importance_scores(q, k, lse_t, cu_q, cu_kv, 1, T, B)
    big = 64
    idx, cnt = O.topk_select(sc, cu_q, cu_kv, T, B, big, w=w, exclusive=True)
    o_s, lse_s = O.sparse_attention(q, k, v, idx, cnt, cu_q, cu_kv, T, B, w)
    assert np.allclose(o_s, o_f, atol=1e-12) and np.allclose(lse_s, lse_f, atol=1e-12)


def test_exclusive_without_candidates_is_the_window_alone():
    # every query of the tile lies within w of the sequence start: no candidate block
    w, T = 8, 4
    cu_q, cu_kv = [0, 6], [0, 6]
    q, k, v = _rand_qkv(cu_q, cu_kv)
    sc = np.ones((2, 1, 6))
    idx, cnt = O.topk_select(sc, cu_q, cu_kv, T, 1, 3, w=w, exclusive=True)
    assert (cnt == 0).all() and (idx == -1).all()
    o_s, _ = O.sparse_attention(q, k, v, idx, cnt, cu_q, cu_kv, T, 1, w)
    o_w, _ = O.swa_attention(q, k, v, cu_q, cu_kv, w)
    assert np.allclose(o_s, o_w, atol=1e-12)
    assert math.isclose(float(np.abs(o_s - o_w).max()), 0.0, abs_tol=1e-12)
