"""fp64 CPU oracle for the hybrid-block attention path (HySparse / HySparse2).

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check of the build entry
point and the CPU-baseline leg of the benchmark import this module. The CUDA
library never calls it, and it shares no code with the CUDA library; the only
common module is the seeded input generator (``workloads``), which holds none
of the arithmetic below.

Every function is the plain definition, evaluated in float64 with numpy.
Matrix products and sorting are library primitives; there is no blocking,
fusion or online rescaling. Work is split only over independent output rows
(one head, one selection tile at a time), which leaves each row's arithmetic
unchanged.

Sources (web pages on the method, cited by page title and paragraph):
  [QbitAI-HySparse]   QbitAI repost "Xiaomi MiMo ... HySparse" -- the hybrid
                      block (1 full layer + N sparse layers reusing its token
                      indices and KV cache) and the two sparse-layer branches
                      (block-sparse global branch, own-cache sliding window of
                      128, fused by a sigmoid gate).
  [techwalker-HySparse] "Xiaomi team launches HySparse ..." -- the master layer
                      computes standard scaled dot-product attention and emits
                      block-level importance from the online-softmax row max
                      (paragraphs "In the concrete implementation" and "the
                      sparse branch concatenates the selected KV blocks ...";
                      the sliding window must keep its own KV).
  [airebao-HySparse2] "Xiaomi MiMo team releases HySparse2" -- KV Reuse of the
                      full layer's KV cache and top-k indices, token-level
                      selection (1024 tokens), the most recent 128 tokens forced
                      into the selected set, MQA, FP8 KV cache (key-data table).
  [demingchina-HySparse2] section 03 -- 1024 global tokens plus the latest 128.
Where the pages leave a step open, the reading used here is stated next to the
function (score formula, tile granularity, GQA max, forced-window union, gate
formula, FP8 scale granularity).

Index conventions
-----------------
* Sequence b has n_b new queries at positions c_b .. c_b + n_b - 1 and
  kv_b = c_b + n_b keys (the new tokens' keys are already in the cache).
  cu_q / cu_kv are prefix sums of n_b / kv_b over the packed token axis.
* Q/O are [T_q, H_q, d]; K/V are [T_kv, H_kv, d]; head h uses KV head h // G.
* Selection tiles: tile i of sequence b covers new queries [i*T, min((i+1)*T, n_b));
  tiles are numbered sequence by sequence.
* Scores are [n_tiles, H_kv, ceil(max_kv / B)]; entries that are not candidates
  are 0. Indices are [n_tiles, H_kv, k] int32, ascending, padded with -1.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bf16 bit patterns: a bf16 is the top half of an IEEE fp32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def e4m3_to_f64(codes) -> np.ndarray:
    """Exact value of OCP FP8 E4M3 codes (1 sign, 4 exponent, 3 mantissa bits,
    bias 7, no infinities, S.1111.111 = NaN, largest finite 448).

    normal (E > 0):  (-1)^S * 2^(E-7) * (1 + M/8)
    subnormal (E=0): (-1)^S * 2^(-6)  * (M/8)
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where(s == 1, -mag, mag)
    return np.where((e == 0xF) & (m == 0x7), np.nan, val)


def dequant_fp8(codes, scale) -> np.ndarray:
    """x = scale_j * e4m3(code): one fp32 scale per (token, KV head)."""
    return e4m3_to_f64(codes) * np.asarray(scale, dtype=np.float64)[..., None]


def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


# ----------------------------------------------------------------------------
# Sequence / tile bookkeeping
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class Tile:
    index: int      # global tile number
    seq: int
    row0: int       # first packed query row (index into T_q)
    n: int          # queries in the tile
    pos0: int       # position of the first query in its sequence
    kv0: int        # first packed key row of the sequence
    kv_len: int     # keys of the sequence

    @property
    def last_pos(self) -> int:
        return self.pos0 + self.n - 1


def make_tiles(cu_q: Sequence[int], cu_kv: Sequence[int], T: int) -> List[Tile]:
    tiles = []
    for b in range(len(cu_q) - 1):
        n_b = cu_q[b + 1] - cu_q[b]
        kv_b = cu_kv[b + 1] - cu_kv[b]
        c_b = kv_b - n_b
        for i in range((n_b + T - 1) // T):
            lo = i * T
            n = min(T, n_b - lo)
            tiles.append(Tile(len(tiles), b, cu_q[b] + lo, n, c_b + lo, cu_kv[b], kv_b))
    return tiles


def softmax_scale(d: int, scale: Optional[float]) -> float:
    # "scaled dot-product attention" [techwalker-HySparse]: 1/sqrt(d)
    return 1.0 / math.sqrt(d) if not scale else float(scale)


# ----------------------------------------------------------------------------
# Masked softmax attention over an explicit visible set
# ----------------------------------------------------------------------------

def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, visible: np.ndarray,
                     scale: float):
    """o_i = sum_j softmax_j(s_ij) v_j over visible j, s_ij = scale * q_i . k_j.

    q [n, d], k/v [m, d], visible [n, m] bool. Returns o [n, d] and
    lse [n] = ln sum_{visible j} exp(s_ij). A row with no visible key has
    o = 0 and lse = -inf.
    """
    s = (q @ k.T) * scale
    s = np.where(visible, s, NEG_INF)
    mx = s.max(axis=1, initial=NEG_INF)
    safe = np.where(np.isfinite(mx), mx, 0.0)
    e = np.where(visible, np.exp(s - safe[:, None]), 0.0)
    tot = e.sum(axis=1)
    with np.errstate(divide="ignore"):
        lse = np.where(tot > 0, safe + np.log(np.where(tot > 0, tot, 1.0)), NEG_INF)
    p = np.where(tot[:, None] > 0, e / np.where(tot > 0, tot, 1.0)[:, None], 0.0)
    return p @ v, lse


# ----------------------------------------------------------------------------
# A1  full causal attention (the full layer) -> O, lse
# ----------------------------------------------------------------------------

def _row_slots(tiles, compact):
    """Output row range of each tile: its packed rows, or consecutive slots when
    only the selected tiles' rows are kept (compact)."""
    out, r = [], 0
    for t in tiles:
        out.append(slice(r, r + t.n) if compact else slice(t.row0, t.row0 + t.n))
        r += t.n
    return out, r


def full_attention(q, k, v, cu_q, cu_kv, n_kv_heads: int, scale=None, tiles_T: int = 0,
                   tile_ids: Optional[Sequence[int]] = None, compact: bool = False):
    """Causal scaled dot-product attention [techwalker-HySparse; QbitAI-HySparse].

    o_{q,h} = sum_{j <= pos(q)} softmax_j(s) v_j,  s = q . k_j / sqrt(d),
    lse_{q,h} = ln sum_{j <= pos(q)} exp(s).

    Returns (o [T_q, H_q, d], lse [H_q, T_q]); with ``tile_ids`` (and tiles_T)
    only those tiles' rows are computed and the rest stay NaN; with
    ``compact`` the outputs hold only those rows, tile after tile.
    """
    Tq, Hq, d = q.shape
    G = Hq // n_kv_heads
    sc = softmax_scale(d, scale)
    T = tiles_T if tiles_T else max(1, max(cu_q[b + 1] - cu_q[b] for b in range(len(cu_q) - 1)))
    tiles = make_tiles(cu_q, cu_kv, T)
    if tile_ids is not None:
        tiles = [tiles[i] for i in tile_ids]
    slots, n_out = _row_slots(tiles, compact)
    o = np.full((n_out if compact else Tq, Hq, d), np.nan)
    lse = np.full((Hq, n_out if compact else Tq), np.nan)
    for t, rows_out in zip(tiles, slots):
        rows = slice(t.row0, t.row0 + t.n)
        pos = t.pos0 + np.arange(t.n)
        kk = k[t.kv0:t.kv0 + t.kv_len]
        vv = v[t.kv0:t.kv0 + t.kv_len]
        vis = np.arange(t.kv_len)[None, :] <= pos[:, None]
        for h in range(Hq):
            g = h // G
            oh, lh = masked_attention(q[rows, h], kk[:, g], vv[:, g], vis, sc)
            o[rows_out, h] = oh
            lse[h, rows_out] = lh
    return o, lse


# ----------------------------------------------------------------------------
# A2  importance scores (by-product of the full layer)
# ----------------------------------------------------------------------------

def importance_scores(q, k, lse, cu_q, cu_kv, n_kv_heads: int, T: int, B: int, scale=None,
                      tile_ids: Optional[Sequence[int]] = None, compact: bool = False):
    """score(t, g, b) = max over queries q in tile t, heads h of KV group g and
    keys j of block b with j <= pos(q) of exp(s_{q,h,j} - lse_{q,h}).

    The pages say the full layer's modified FlashAttention emits block-level
    maximum attention scores from the online-softmax row maximum
    [techwalker-HySparse]; the maximum is taken over the tile's queries and the
    group's heads (reading), with tile T from the workload. A block b is a
    candidate of tile t iff b*B <= last position of t; non-candidates are 0.

    Returns scores [n_tiles, H_kv, ceil(max_kv/B)] (rows not in tile_ids stay 0).
    ``lse`` is indexed like full_attention's output (compact rows if compact);
    with ``compact`` the scores hold only the selected tiles, in order.
    """
    Tq, Hq, d = q.shape
    G = Hq // n_kv_heads
    sc = softmax_scale(d, scale)
    tiles = make_tiles(cu_q, cu_kv, T)
    max_kv = max(cu_kv[b + 1] - cu_kv[b] for b in range(len(cu_kv) - 1))
    nblk = (max_kv + B - 1) // B
    sel = tiles if tile_ids is None else [tiles[i] for i in tile_ids]
    slots, _ = _row_slots(sel, compact)
    scores = np.zeros((len(sel) if compact else len(tiles), n_kv_heads, nblk))
    for si, (t, rows_out) in enumerate(zip(sel, slots)):
        out_i = si if compact else t.index
        n_cand_keys = min(t.kv_len, (t.last_pos // B + 1) * B)
        pos = t.pos0 + np.arange(t.n)
        vis = np.arange(n_cand_keys)[None, :] <= pos[:, None]
        for g in range(n_kv_heads):
            kk = k[t.kv0:t.kv0 + n_cand_keys, g]
            colmax = np.zeros(n_cand_keys)
            for h in range(g * G, (g + 1) * G):
                s = (q[t.row0:t.row0 + t.n, h] @ kk.T) * sc
                p = np.where(vis, np.exp(s - lse[h, rows_out][:, None]), 0.0)
                colmax = np.maximum(colmax, p.max(axis=0))
            nb = (n_cand_keys + B - 1) // B
            padded = np.zeros(nb * B)
            padded[:n_cand_keys] = colmax
            scores[out_i, g, :nb] = padded.reshape(nb, B).max(axis=1)
    return scores


# ----------------------------------------------------------------------------
# A3  top-k selection
# ----------------------------------------------------------------------------

def n_candidates(t: Tile, B: int, w: int = 0, exclusive: bool = False) -> int:
    """Candidate blocks of a tile.

    Union reading (default): every causal block, b*B <= last query position;
    the forced window is added per query afterwards, so a selected block may
    overlap it [airebao-HySparse2: the latest tokens are forced into the
    selected set].
    Exclusive reading: only blocks that start before the forced window of the
    tile's last query, b*B <= last_pos - w, compete, so the k selected blocks
    are "global" tokens and the w recent ones come on top
    [demingchina-HySparse2 s.03: 1024 global tokens plus the latest 128].
    With w = 0 the two readings coincide.
    """
    if not exclusive:
        return t.last_pos // B + 1
    lim = t.last_pos - w
    return 0 if lim < 0 else lim // B + 1


def topk_select(scores, cu_q, cu_kv, T: int, B: int, k: int,
                tile_ids: Optional[Sequence[int]] = None, compact: bool = False,
                w: int = 0, exclusive: bool = False):
    """Keep the k highest-scoring candidate blocks of each (tile, KV head).

    Candidates per n_candidates (union or exclusive reading of the forced
    window). Order: score descending, ties to the lower block index (the
    reading used throughout; the pages only say "TopK"). The kept set is
    emitted in ascending index order and padded with -1;
    cnt = min(k, #candidates).
    Returns (idx int32 [n_tiles, H_kv, k], cnt int32 [n_tiles, H_kv]).
    """
    n_rows, Hkv, _ = scores.shape
    tiles = make_tiles(cu_q, cu_kv, T)
    idx = np.full((n_rows, Hkv, k), -1, dtype=np.int32)
    cnt = np.zeros((n_rows, Hkv), dtype=np.int32)
    sel = tiles if tile_ids is None else [tiles[i] for i in tile_ids]
    for si, t in enumerate(sel):
        r = si if compact else t.index   # compact: scores/idx rows follow tile_ids
        nc = n_candidates(t, B, w, exclusive)
        ids = np.arange(nc)
        for g in range(Hkv):
            s = scores[r, g, :nc]
            order = np.lexsort((ids, -s))          # primary: -score, secondary: index
            keep = np.sort(order[:min(k, nc)])
            idx[r, g, :len(keep)] = keep
            cnt[r, g] = len(keep)
    return idx, cnt


# ----------------------------------------------------------------------------
# A4 / A6  sparse attention over the reused KV cache and indices
# ----------------------------------------------------------------------------

def sparse_visible(t: Tile, sel_blocks: Sequence[int], B: int, w: int) -> np.ndarray:
    """Visible keys of each query of a tile, as a bool matrix [t.n, kv_len].

    V_q = {j in blocks(idx_t) : j <= q - w}  union  [max(0, q - w + 1), q].
    The recent w tokens are forced into the selected set [airebao-HySparse2;
    demingchina-HySparse2 s.03]; reading: the union is taken per query and a
    selected key inside the window is counted once. w = 0 gives the plain
    causal block-sparse branch of HySparse [QbitAI-HySparse].
    """
    pos = t.pos0 + np.arange(t.n)
    in_sel = np.zeros(t.kv_len, dtype=bool)
    for b in sel_blocks:
        if b < 0:
            continue
        in_sel[b * B:min((b + 1) * B, t.kv_len)] = True
    j = np.arange(t.kv_len)[None, :]
    from_sel = in_sel[None, :] & (j <= pos[:, None] - w)
    from_win = (j >= np.maximum(0, pos[:, None] - w + 1)) & (j <= pos[:, None])
    return from_sel | from_win


def sparse_attention(q, k, v, idx, cnt, cu_q, cu_kv, T: int, B: int, w: int, scale=None,
                     tile_ids: Optional[Sequence[int]] = None, compact: bool = False):
    """Sparse layer: softmax attention of this layer's Q over V_q, using the
    full layer's K/V and its tile indices (KV Reuse) [QbitAI-HySparse;
    airebao-HySparse2]. Returns (o [T_q, H_q, d], lse [H_q, T_q]); tiles not in
    tile_ids stay NaN. An empty V_q (possible only with w = 0) gives o = 0,
    lse = -inf.
    """
    Tq, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    sc = softmax_scale(d, scale)
    tiles = make_tiles(cu_q, cu_kv, T)
    sel = tiles if tile_ids is None else [tiles[i] for i in tile_ids]
    slots, n_out = _row_slots(sel, compact)
    o = np.full((n_out if compact else Tq, Hq, d), np.nan)
    lse = np.full((Hq, n_out if compact else Tq), np.nan)
    for si, (t, rows_out) in enumerate(zip(sel, slots)):
        rows = slice(t.row0, t.row0 + t.n)
        r = si if compact else t.index   # compact: idx/cnt rows follow tile_ids
        for g in range(Hkv):
            vis = sparse_visible(t, idx[r, g, :cnt[r, g]], B, w)
            cols = np.nonzero(vis.any(axis=0))[0]
            kk = k[t.kv0 + cols, g]
            vv = v[t.kv0 + cols, g]
            for h in range(g * G, (g + 1) * G):
                oh, lh = masked_attention(q[rows, h], kk, vv, vis[:, cols], sc)
                o[rows_out, h] = oh
                lse[h, rows_out] = lh
    return o, lse


# ----------------------------------------------------------------------------
# A5  sliding-window branch with its own KV, and the sigmoid gate
# ----------------------------------------------------------------------------

def swa_attention(q, k_swa, v_swa, cu_q, cu_kv, window: int, scale=None,
                  row_ids: Optional[Sequence[int]] = None, compact: bool = False):
    """SWA branch of a HySparse sparse layer: same Q, its own small KV cache,
    keys [max(0, q - window + 1), q] (window 128 by default)
    [QbitAI-HySparse; techwalker-HySparse]. Returns (o, lse [H_q, T_q])."""
    Tq, Hq, d = q.shape
    Hkv = k_swa.shape[1]
    G = Hq // Hkv
    sc = softmax_scale(d, scale)
    rows_all = list(range(Tq)) if row_ids is None else list(row_ids)
    n_out = len(rows_all) if compact else Tq
    o = np.full((n_out, Hq, d), np.nan)
    lse = np.full((Hq, n_out), np.nan)
    cu = np.asarray(cu_q)
    for ri, r in enumerate(rows_all):
        ro = ri if compact else r
        b = int(np.searchsorted(cu, r, side="right") - 1)
        n_b = cu_q[b + 1] - cu_q[b]
        kv_b = cu_kv[b + 1] - cu_kv[b]
        p = kv_b - n_b + (r - cu_q[b])
        lo = max(0, p - window + 1)
        keys = slice(cu_kv[b] + lo, cu_kv[b] + p + 1)
        vis = np.ones((1, p + 1 - lo), dtype=bool)
        for h in range(Hq):
            g = h // G
            oh, lh = masked_attention(q[r:r + 1, h], k_swa[keys, g], v_swa[keys, g], vis, sc)
            o[ro, h] = oh[0]
            lse[h, ro] = lh[0]
    return o, lse


def gated_merge(gamma, o_sparse, o_swa):
    """o = sigmoid(gamma) * o_sparse + (1 - sigmoid(gamma)) * o_swa, gamma per
    (token, head). The pages name only a sigmoid gate fusing the two branches
    [QbitAI-HySparse; techwalker-HySparse]; this convex form is the reading."""
    s = sigmoid(gamma)[..., None]
    return s * o_sparse + (1.0 - s) * o_swa
