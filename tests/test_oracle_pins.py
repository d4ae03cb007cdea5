"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each test checks the oracle against one of: a closed form, an exhaustive
enumeration on tiny inputs written as plain Python loops (a different route
from the oracle's matrix code), an invariant of the method stated by its
definition, a textbook special case, or an independent library decoder.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(7)


# ---------------------------------------------------------------- number formats

@pytest.mark.filterwarnings("ignore:invalid value encountered in cast:RuntimeWarning")  # NaN patterns
def test_bf16_decode_matches_torch_for_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_bf16_decode_known_values():
    assert O.bf16_to_f64([0x3F80])[0] == 1.0
    assert O.bf16_to_f64([0xC000])[0] == -2.0
    assert O.bf16_to_f64([0x0001])[0] == 2.0 ** -133
    assert O.bf16_to_f64([0x7F7F])[0] == (2 - 2 ** -7) * 2.0 ** 127


def test_e4m3_known_values_from_format_definition():
    # OCP 8-bit floating point spec, E4M3: bias 7, max normal S.1111.110 = 448,
    # min normal 2^-6, min subnormal 2^-9, S.1111.111 = NaN, no infinities.
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x3C: 1.5, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0, 0x80: -0.0,
             0xB8: -1.0}
    got = O.e4m3_to_f64(list(table.keys()))
    assert list(got) == list(table.values())
    assert np.isnan(O.e4m3_to_f64([0x7F, 0xFF])).all()


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_fp8_round_trip_error_bound():
    from workloads import quantize_e4m3_per_token
    x = torch.randn(64, 2, 128, generator=torch.Generator().manual_seed(3))
    codes, scale = quantize_e4m3_per_token(x)
    back = O.dequant_fp8(codes.numpy(), scale.numpy())
    # e4m3 has 3 mantissa bits: relative rounding error <= 2^-4 for normals;
    # subnormals (|y| < 2^-6 in units of scale) have absolute error <= 2^-10 * scale.
    err = np.abs(back - x.double().numpy())
    bound = np.maximum(np.abs(x.double().numpy()) * 2 ** -4, 2.0 ** -10 * scale.double().numpy()[..., None])
    assert (err <= bound * (1 + 1e-12)).all()


# ---------------------------------------------------------------- masked attention

def _online_attention_row(q, ks, vs, scale):
    """Attention for one row by sequential accumulation in plain Python
    (running max and running sum): a different route from the oracle's
    matrix/logsumexp code."""
    m = -math.inf
    l = 0.0
    acc = [0.0] * len(vs[0])
    for kj, vj in zip(ks, vs):
        s = scale * sum(a * b for a, b in zip(q, kj))
        m_new = max(m, s)
        c = math.exp(m - m_new) if m != -math.inf else 0.0
        p = math.exp(s - m_new)
        l = l * c + p
        acc = [a * c + p * b for a, b in zip(acc, vj)]
        m = m_new
    return [a / l for a in acc], m + math.log(l)


def test_masked_attention_matches_sequential_accumulation():
    n, m, d = 5, 9, 6
    q = RNG.standard_normal((n, d))
    k = RNG.standard_normal((m, d)) * 2
    v = RNG.standard_normal((m, d))
    vis = RNG.random((n, m)) < 0.6
    vis[:, 0] = True
    o, lse = O.masked_attention(q, k, v, vis, 0.37)
    for i in range(n):
        cols = [j for j in range(m) if vis[i, j]]
        ro, rl = _online_attention_row(q[i], k[cols], v[cols], 0.37)
        assert np.allclose(o[i], ro, rtol=0, atol=1e-12)
        assert abs(lse[i] - rl) < 1e-12


def test_masked_attention_empty_row():
    o, lse = O.masked_attention(np.ones((1, 2)), np.ones((3, 2)), np.ones((3, 2)),
                                np.zeros((1, 3), dtype=bool), 1.0)
    assert (o == 0).all() and lse[0] == -np.inf


def test_softmax_closed_form_golden():
    """Hand-derived example in tests/golden/softmax_closed_form.json."""
    with open(os.path.join(GOLDEN, "softmax_closed_form.json")) as f:
        g = json.load(f)
    q = np.array(g["q"], dtype=np.float64)[None, None, :]
    k = np.array(g["k"], dtype=np.float64)[:, None, :]
    v = np.array(g["v"], dtype=np.float64)[:, None, :]
    cu = [0, 1]
    cukv = [0, len(g["k"])]
    o, lse = O.full_attention(q, k, v, cu, cukv, 1)
    assert np.allclose(o[0, 0], g["o"], atol=1e-12)
    assert abs(lse[0, 0] - math.log(g["lse_exp"])) < 1e-12


# ---------------------------------------------------------------- full attention

def _rand_case(Hq=4, Hkv=2, d=8, new=(7, 5), ctx=(3, 0)):
    kv = [c + n for c, n in zip(ctx, new)]
    cu_q = [0] + list(np.cumsum(new))
    cu_kv = [0] + list(np.cumsum(kv))
    q = RNG.standard_normal((cu_q[-1], Hq, d))
    k = RNG.standard_normal((cu_kv[-1], Hkv, d))
    v = RNG.standard_normal((cu_kv[-1], Hkv, d))
    return q, k, v, [int(x) for x in cu_q], [int(x) for x in cu_kv]


def test_full_attention_zero_query_is_causal_mean():
    q, k, v, cu_q, cu_kv = _rand_case()
    q[:] = 0.0
    o, lse = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    G = 2
    for b in range(2):
        n_b = cu_q[b + 1] - cu_q[b]
        kv_b = cu_kv[b + 1] - cu_kv[b]
        for i in range(n_b):
            p = kv_b - n_b + i
            for h in range(4):
                want = v[cu_kv[b]:cu_kv[b] + p + 1, h // G].mean(axis=0)
                assert np.allclose(o[cu_q[b] + i, h], want, atol=1e-12)
                assert abs(lse[h, cu_q[b] + i] - math.log(p + 1)) < 1e-12


def test_full_attention_first_position_returns_v0():
    q, k, v, cu_q, cu_kv = _rand_case(ctx=(0, 0))
    o, lse = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    for b in range(2):
        r = cu_q[b]
        for h in range(4):
            assert np.array_equal(o[r, h], v[cu_kv[b], h // 2])
            s0 = q[r, h] @ k[cu_kv[b], h // 2] / math.sqrt(8)
            assert abs(lse[h, r] - s0) < 1e-12


def test_full_attention_gqa_head_mapping():
    q, k, v, cu_q, cu_kv = _rand_case(Hq=6, Hkv=3)
    for g in range(3):
        v[:, g, :] = g + 1.0
    o, _ = O.full_attention(q, k, v, cu_q, cu_kv, 3)
    for h in range(6):
        assert np.allclose(o[:, h], h // 2 + 1.0, atol=1e-12)


def test_full_attention_matches_loops_and_lse_bounds():
    q, k, v, cu_q, cu_kv = _rand_case()
    o, lse = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    sc = 1 / math.sqrt(8)
    for b in range(2):
        n_b = cu_q[b + 1] - cu_q[b]
        kv_b = cu_kv[b + 1] - cu_kv[b]
        for i in range(n_b):
            p = kv_b - n_b + i
            r = cu_q[b] + i
            for h in range(4):
                ks = k[cu_kv[b]:cu_kv[b] + p + 1, h // 2]
                vs = v[cu_kv[b]:cu_kv[b] + p + 1, h // 2]
                ro, rl = _online_attention_row(q[r, h], ks, vs, sc)
                assert np.allclose(o[r, h], ro, atol=1e-12)
                assert abs(lse[h, r] - rl) < 1e-12
                mx = max(sc * (q[r, h] @ kk) for kk in ks)
                assert mx - 1e-12 <= lse[h, r] <= mx + math.log(p + 1) + 1e-12


def test_rows_sum_to_one():
    q, k, v, cu_q, cu_kv = _rand_case()
    v[:] = 1.0
    o, _ = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    assert np.allclose(o, 1.0, atol=1e-12)


# ---------------------------------------------------------------- scores

def _brute_scores(q, k, cu_q, cu_kv, Hkv, T, B):
    """Enumerate every (query, head, key) triple with plain loops; lse by a
    plain Python sum of exponentials."""
    Tq, Hq, d = q.shape
    G = Hq // Hkv
    sc = 1 / math.sqrt(d)
    tiles = O.make_tiles(cu_q, cu_kv, T)
    max_kv = max(cu_kv[i + 1] - cu_kv[i] for i in range(len(cu_kv) - 1))
    out = np.zeros((len(tiles), Hkv, (max_kv + B - 1) // B))
    for t in tiles:
        for qi in range(t.n):
            p = t.pos0 + qi
            r = t.row0 + qi
            for h in range(Hq):
                g = h // G
                logits = [sc * sum(q[r, h, e] * k[t.kv0 + j, g, e] for e in range(d))
                          for j in range(p + 1)]
                lse = math.log(sum(math.exp(x) for x in logits))
                for j in range(p + 1):
                    val = math.exp(logits[j] - lse)
                    out[t.index, g, j // B] = max(out[t.index, g, j // B], val)
    return out


@pytest.mark.parametrize("T,B", [(4, 2), (3, 1), (5, 4)])
def test_scores_match_enumeration(T, B):
    q, k, v, cu_q, cu_kv = _rand_case(new=(9, 6), ctx=(2, 0), d=4)
    _, lse = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    got = O.importance_scores(q, k, lse, cu_q, cu_kv, 2, T, B)
    want = _brute_scores(q, k, cu_q, cu_kv, 2, T, B)
    assert np.allclose(got, want, rtol=1e-12, atol=0)


def test_score_is_one_only_for_single_key_rows():
    q, k, v, cu_q, cu_kv = _rand_case(ctx=(0, 0), new=(8,))
    cu_q, cu_kv = [0, 8], [0, 8]
    _, lse = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    sc = O.importance_scores(q, k, lse, cu_q, cu_kv, 2, 4, 2)
    assert (sc <= 1 + 1e-15).all()
    # position 0 sees only key 0, so block 0 of tile 0 scores exactly 1
    assert np.allclose(sc[0, :, 0], 1.0, atol=1e-15)
    # tile 1 (positions 4..7) sees >= 5 keys per row: every score < 1
    assert (sc[1] < 1).all()


def test_planted_key_is_top_scored():
    d, L = 16, 64
    q = RNG.standard_normal((L, 1, d))
    k = RNG.standard_normal((L, 1, d))
    v = RNG.standard_normal((L, 1, d))
    j, p = 10, 40
    k[j, 0] = 4 * math.sqrt(d) * q[p, 0] / np.linalg.norm(q[p, 0])
    _, lse = O.full_attention(q, k, v, [0, L], [0, L], 1)
    sc = O.importance_scores(q, k, lse, [0, L], [0, L], 1, 16, 1)
    t = p // 16
    assert int(np.argmax(sc[t, 0])) == j


# ---------------------------------------------------------------- top-k

def _is_valid_selection(s, sel, k):
    n = len(s)
    if len(sel) != min(k, n):
        return False
    rest = [j for j in range(n) if j not in sel]
    return all(s[i] > s[j] or (s[i] == s[j] and i < j) for i in sel for j in rest)


@pytest.mark.parametrize("trial", range(6))
def test_topk_unique_valid_subset(trial):
    rng = np.random.default_rng(100 + trial)
    T, B, k = 4, 1, 4
    L = 9
    cu = [0, L]
    tiles = O.make_tiles(cu, cu, T)
    nblk = L
    scores = np.zeros((len(tiles), 1, nblk))
    for t in tiles:
        nc = O.n_candidates(t, B)
        scores[t.index, 0, :nc] = rng.integers(1, 4, nc) / 4.0  # many ties
    idx, cnt = O.topk_select(scores, cu, cu, T, B, k)
    for t in tiles:
        nc = O.n_candidates(t, B)
        s = list(scores[t.index, 0, :nc])
        valid = [set(c) for c in itertools.combinations(range(nc), min(k, nc))
                 if _is_valid_selection(s, set(c), k)]
        assert len(valid) == 1
        got = idx[t.index, 0]
        assert cnt[t.index, 0] == min(k, nc)
        assert list(got[:cnt[t.index, 0]]) == sorted(valid[0])
        assert (got[cnt[t.index, 0]:] == -1).all()


def test_topk_all_equal_takes_lowest_indices():
    cu = [0, 20]
    scores = np.zeros((1, 1, 20))
    scores[0, 0, :] = 0.5
    idx, cnt = O.topk_select(scores, cu, cu, 20, 1, 5)
    assert list(idx[0, 0]) == [0, 1, 2, 3, 4] and cnt[0, 0] == 5


def test_topk_distinct_matches_argsort():
    cu = [0, 64]
    s = RNG.permutation(64).astype(np.float64) + 1
    scores = s.reshape(1, 1, 64)
    idx, _ = O.topk_select(scores, cu, cu, 64, 1, 10)
    assert list(idx[0, 0]) == sorted(np.argsort(-s, kind="stable")[:10].tolist())


def test_topk_respects_causal_candidates():
    cu = [0, 8]
    scores = np.ones((2, 1, 8))
    idx, cnt = O.topk_select(scores, cu, cu, 4, 2, 8)
    # tile 0: last position 3 -> blocks 0..1; tile 1: last position 7 -> blocks 0..3
    assert cnt[0, 0] == 2 and list(idx[0, 0, :3]) == [0, 1, -1]
    assert cnt[1, 0] == 4 and list(idx[1, 0, :5]) == [0, 1, 2, 3, -1]


# ---------------------------------------------------------------- sparse / SWA / gate

def _visible_by_definition(p, blocks, B, w):
    """V_p from its definition, as a Python set."""
    sel = set()
    for b in blocks:
        for j in range(b * B, b * B + B):
            if j <= p - w:
                sel.add(j)
    win = set(range(max(0, p - w + 1), p + 1))
    return sel | win


@pytest.mark.parametrize("B,w", [(2, 3), (1, 4), (4, 0), (3, 1)])
def test_sparse_zero_query_is_mean_over_visible_set(B, w):
    q, k, v, cu_q, cu_kv = _rand_case(new=(10, 7), ctx=(5, 2), Hq=2, Hkv=1)
    q[:] = 0.0
    T, topk = 4, 2
    _, lse = O.full_attention(RNG.standard_normal(q.shape), k, v, cu_q, cu_kv, 1)
    tiles = O.make_tiles(cu_q, cu_kv, T)
    nb = max(cu_kv[i + 1] - cu_kv[i] for i in range(2)) // B + 1
    idx = np.full((len(tiles), 1, topk), -1, dtype=np.int32)
    cnt = np.zeros((len(tiles), 1), dtype=np.int32)
    for t in tiles:
        nc = O.n_candidates(t, B)
        chosen = sorted(RNG.choice(nc, size=min(topk, nc), replace=False).tolist())
        idx[t.index, 0, :len(chosen)] = chosen
        cnt[t.index, 0] = len(chosen)
    o, lse_s = O.sparse_attention(q, k, v, idx, cnt, cu_q, cu_kv, T, B, w)
    for t in tiles:
        for i in range(t.n):
            p = t.pos0 + i
            vis = _visible_by_definition(p, idx[t.index, 0, :cnt[t.index, 0]], B, w)
            vis = sorted(j for j in vis if j < t.kv_len)
            for h in range(2):
                r = t.row0 + i
                if not vis:
                    assert (o[r, h] == 0).all() and lse_s[h, r] == -np.inf
                else:
                    want = v[t.kv0 + np.array(vis), 0].mean(axis=0)
                    assert np.allclose(o[r, h], want, atol=1e-12)
                    assert abs(lse_s[h, r] - math.log(len(vis))) < 1e-12


@pytest.mark.parametrize("w", [0, 3])
def test_sparse_with_all_candidates_equals_full(w):
    q, k, v, cu_q, cu_kv = _rand_case()
    T, B = 3, 2
    o_f, lse_f = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    big = 100
    scores = np.ones((len(O.make_tiles(cu_q, cu_kv, T)), 2, big))
    idx, cnt = O.topk_select(scores, cu_q, cu_kv, T, B, big)
    o_s, lse_s = O.sparse_attention(q, k, v, idx, cnt, cu_q, cu_kv, T, B, w)
    assert np.allclose(o_s, o_f, atol=1e-12) and np.allclose(lse_s, lse_f, atol=1e-12)


def test_sparse_with_k0_equals_swa_window():
    q, k, v, cu_q, cu_kv = _rand_case()
    T, B, w = 3, 2, 3
    n_t = len(O.make_tiles(cu_q, cu_kv, T))
    idx = np.full((n_t, 2, 1), -1, dtype=np.int32)
    cnt = np.zeros((n_t, 2), dtype=np.int32)
    o_s, lse_s = O.sparse_attention(q, k, v, idx, cnt, cu_q, cu_kv, T, B, w)
    o_w, lse_w = O.swa_attention(q, k, v, cu_q, cu_kv, w)
    assert np.allclose(o_s, o_w, atol=1e-12) and np.allclose(lse_s, lse_w, atol=1e-12)


def test_swa_with_wide_window_equals_full():
    q, k, v, cu_q, cu_kv = _rand_case()
    o_f, lse_f = O.full_attention(q, k, v, cu_q, cu_kv, 2)
    o_w, lse_w = O.swa_attention(q, k, v, cu_q, cu_kv, 1000)
    assert np.allclose(o_w, o_f, atol=1e-12) and np.allclose(lse_w, lse_f, atol=1e-12)


def test_swa_window_one_returns_own_value():
    q, k, v, cu_q, cu_kv = _rand_case()
    o_w, _ = O.swa_attention(q, k, v, cu_q, cu_kv, 1)
    for b in range(2):
        n_b = cu_q[b + 1] - cu_q[b]
        kv_b = cu_kv[b + 1] - cu_kv[b]
        for i in range(n_b):
            p = kv_b - n_b + i
            for h in range(4):
                assert np.array_equal(o_w[cu_q[b] + i, h], v[cu_kv[b] + p, h // 2])


def test_gate_extremes_and_midpoint():
    a = RNG.standard_normal((3, 2, 4))
    b = RNG.standard_normal((3, 2, 4))
    assert np.allclose(O.gated_merge(np.full((3, 2), 50.0), a, b), a, atol=1e-15)
    assert np.allclose(O.gated_merge(np.full((3, 2), -50.0), a, b), b, atol=1e-15)
    assert np.allclose(O.gated_merge(np.zeros((3, 2)), a, b), (a + b) / 2, atol=1e-15)
    assert abs(O.sigmoid(math.log(3.0)) - 0.75) < 1e-15
