"""Pins of the oracle's sampled mode (``tile_ids`` / ``compact`` / ``row_ids``).

Full-size parity tests run the oracle on a few selection tiles only. These
CPU tests pin that mode to the all-tiles mode, which the other oracle pins tie
to closed forms and brute force: on ragged chunked batches (one and several
sequences, MQA and GQA, with and without a forced window, block and token
level), every sampled output must equal the matching rows of the all-tiles
call exactly, and the rows of a tile must be the ones a plain scan of the
packed token axis assigns to it.
"""
import numpy as np
import pytest

import oracle as O
from oracle.block import run_block, tile_rows

CASES = {
    # name: (ctx, new, Hq, Hkv, d, T, B, k, w, swa)
    "one_seq_gqa_block_w0": ((0,), (37,), 4, 2, 8, 8, 4, 3, 0, 6),
    "batch_mqa_token_w": ((5, 0, 13), (11, 9, 17), 4, 1, 8, 4, 1, 5, 3, 0),
    "batch_gqa_block_w": ((0, 21), (19, 14), 6, 3, 4, 5, 2, 2, 4, 5),
    "batch_mha_chunked": ((40, 3), (6, 10), 2, 2, 4, 3, 8, 2, 0, 4),
}


def _case(name, seed=0):
    ctx, new, Hq, Hkv, d, T, B, k, w, swa = CASES[name]
    rng = np.random.default_rng(seed)
    kv = [c + n for c, n in zip(ctx, new)]
    cu_q = [0] + [int(x) for x in np.cumsum(new)]
    cu_kv = [0] + [int(x) for x in np.cumsum(kv)]
    q = rng.standard_normal((cu_q[-1], Hq, d))
    kk = rng.standard_normal((cu_kv[-1], Hkv, d))
    v = rng.standard_normal((cu_kv[-1], Hkv, d))
    q2 = rng.standard_normal((cu_q[-1], Hq, d))
    ks = rng.standard_normal((cu_kv[-1], Hkv, d))
    vs = rng.standard_normal((cu_kv[-1], Hkv, d))
    gamma = rng.standard_normal((cu_q[-1], Hq))
    return dict(q=q, k=kk, v=v, q2=q2, ks=ks, vs=vs, gamma=gamma, cu_q=cu_q, cu_kv=cu_kv, Hkv=Hkv, T=T, B=B,
                topk=k, w=w, swa=swa)


def _rows_by_scan(cu_q, T, tile_ids):
    """Packed rows of the given tiles, found by walking the token axis: row r
    of sequence b belongs to tile (tiles before b) + (r - cu_q[b]) // T."""
    owner = []
    before = 0
    for b in range(len(cu_q) - 1):
        n_b = cu_q[b + 1] - cu_q[b]
        for i in range(n_b):
            owner.append(before + i // T)
        before += -(-n_b // T)
    rows = []
    for t in tile_ids:
        rows.extend(r for r in range(cu_q[-1]) if owner[r] == t)
    return rows


def _samples(n_tiles, rng):
    """Tile subsets: every tile, first + last, a random sorted subset and an
    unsorted one."""
    out = [list(range(n_tiles)), sorted({0, n_tiles - 1})]
    if n_tiles > 2:
        out.append(sorted(rng.choice(n_tiles, size=max(1, n_tiles // 2), replace=False).tolist()))
        perm = rng.permutation(n_tiles)[:max(2, n_tiles // 3)].tolist()
        out.append(perm)
    return out


@pytest.mark.parametrize("name", list(CASES))
def test_tile_rows_match_a_scan_of_the_token_axis(name):
    c = _case(name)
    n_t = len(O.make_tiles(c["cu_q"], c["cu_kv"], c["T"]))
    rng = np.random.default_rng(1)
    for ids in _samples(n_t, rng):
        assert tile_rows(c["cu_q"], c["cu_kv"], c["T"], ids) == _rows_by_scan(c["cu_q"], c["T"], ids)


@pytest.mark.parametrize("name", list(CASES))
def test_sampled_outputs_equal_the_all_tiles_rows(name):
    c = _case(name)
    cu_q, cu_kv, Hkv, T, B, k, w = c["cu_q"], c["cu_kv"], c["Hkv"], c["T"], c["B"], c["topk"], c["w"]
    q, kk, v = c["q"], c["k"], c["v"]
    o_all, lse_all = O.full_attention(q, kk, v, cu_q, cu_kv, Hkv, tiles_T=T)
    sc_all = O.importance_scores(q, kk, lse_all, cu_q, cu_kv, Hkv, T, B)
    idx_all, cnt_all = O.topk_select(sc_all, cu_q, cu_kv, T, B, k)
    sp_all, sl_all = O.sparse_attention(c["q2"], kk, v, idx_all, cnt_all, cu_q, cu_kv, T, B, w)
    sw_all, swl_all = O.swa_attention(c["q2"], c["ks"], c["vs"], cu_q, cu_kv, max(c["swa"], 1))
    n_t = len(O.make_tiles(cu_q, cu_kv, T))
    rng = np.random.default_rng(2)
    for ids in _samples(n_t, rng):
        rows = _rows_by_scan(cu_q, T, ids)
        # A1, compact: the sampled tiles' rows, tile after tile
        o_c, lse_c = O.full_attention(q, kk, v, cu_q, cu_kv, Hkv, tiles_T=T, tile_ids=ids, compact=True)
        assert np.array_equal(o_c, o_all[rows]) and np.array_equal(lse_c, lse_all[:, rows])
        # A1, in place: sampled rows filled, every other row left NaN
        o_p, lse_p = O.full_attention(q, kk, v, cu_q, cu_kv, Hkv, tiles_T=T, tile_ids=ids)
        assert np.array_equal(o_p[rows], o_all[rows]) and np.array_equal(lse_p[:, rows], lse_all[:, rows])
        others = sorted(set(range(cu_q[-1])) - set(rows))
        assert np.isnan(o_p[others]).all() and np.isnan(lse_p[:, others]).all()
        # A2 (fed the compact lse) and A3, compact
        sc_c = O.importance_scores(q, kk, lse_c, cu_q, cu_kv, Hkv, T, B, tile_ids=ids, compact=True)
        assert np.array_equal(sc_c, sc_all[ids])
        idx_c, cnt_c = O.topk_select(sc_c, cu_q, cu_kv, T, B, k, tile_ids=ids, compact=True)
        assert np.array_equal(idx_c, idx_all[ids]) and np.array_equal(cnt_c, cnt_all[ids])
        # A2 in place: the sampled tiles' rows of the score tensor, the rest 0
        sc_p = O.importance_scores(q, kk, lse_all, cu_q, cu_kv, Hkv, T, B, tile_ids=ids)
        assert np.array_equal(sc_p[ids], sc_all[ids])
        assert not sc_p[sorted(set(range(n_t)) - set(ids))].any()
        # A4, compact, with the compact indices
        sp_c, sl_c = O.sparse_attention(c["q2"], kk, v, idx_c, cnt_c, cu_q, cu_kv, T, B, w, tile_ids=ids,
                                        compact=True)
        assert np.array_equal(sp_c, sp_all[rows]) and np.array_equal(sl_c, sl_all[:, rows])
        # A5 window branch on the sampled rows
        sw_c, swl_c = O.swa_attention(c["q2"], c["ks"], c["vs"], cu_q, cu_kv, max(c["swa"], 1), row_ids=rows,
                                      compact=True)
        assert np.array_equal(sw_c, sw_all[rows]) and np.array_equal(swl_c, swl_all[:, rows])


@pytest.mark.parametrize("name", list(CASES))
def test_block_on_sampled_tiles_equals_the_whole_block(name):
    c = _case(name)
    cu_q, cu_kv = c["cu_q"], c["cu_kv"]
    layers = [{"q": c["q2"], "k_swa": c["ks"], "v_swa": c["vs"], "gamma": c["gamma"]}]
    args = (c["q"], c["k"], c["v"], layers, cu_q, cu_kv, c["Hkv"], c["T"], c["B"], c["topk"], c["w"], c["swa"])
    whole = run_block(*args)
    n_t = len(O.make_tiles(cu_q, cu_kv, c["T"]))
    ids = sorted({0, n_t - 1, n_t // 2})
    part = run_block(*args, tile_ids=ids)
    rows = _rows_by_scan(cu_q, c["T"], ids)
    assert np.array_equal(part["o_full"][rows], whole["o_full"][rows])
    assert np.array_equal(part["scores"][ids], whole["scores"][ids])
    assert np.array_equal(part["idx"][ids], whole["idx"][ids])
    for a, b in zip(part["layers"], whole["layers"]):
        assert np.array_equal(a["o"][rows], b["o"][rows])
        assert np.array_equal(a["lse_sparse"][:, rows], b["lse_sparse"][:, rows])
    # compact outputs: the same rows, tile after tile
    comp = run_block(*args, tile_ids=ids, compact=True)
    assert np.array_equal(comp["o_full"], whole["o_full"][rows])
    assert np.array_equal(comp["lse_full"], whole["lse_full"][:, rows])
    assert np.array_equal(comp["scores"], whole["scores"][ids])
    assert np.array_equal(comp["idx"], whole["idx"][ids]) and np.array_equal(comp["cnt"], whole["cnt"][ids])
    for a, b in zip(comp["layers"], whole["layers"]):
        assert np.array_equal(a["o"], b["o"][rows]) and np.array_equal(a["o_sparse"], b["o_sparse"][rows])
