"""Whole hybrid block through the fp64 oracle (test infrastructure only).

One full layer (A1 output + lse, A2 scores, A3 indices) feeding N sparse
layers (A4 sparse attention over the reused K/V and indices; for HySparse also
the A5 own-cache SWA branch and the sigmoid gate), evaluated on a subset of
selection tiles so that full-size workloads can be checked on samples.
Inputs are numpy arrays already decoded to float64 (see ``bf16_to_f64``).
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from . import hs_oracle as O


def tile_rows(cu_q, cu_kv, T, tile_ids):
    tiles = O.make_tiles(cu_q, cu_kv, T)
    rows = []
    for i in tile_ids:
        t = tiles[i]
        rows.extend(range(t.row0, t.row0 + t.n))
    return rows


def run_block(q, k, v, layers, cu_q, cu_kv, n_kv_heads, T, B, topk, w, swa_window=0,
              tile_ids: Optional[Sequence[int]] = None, idx_override=None, cnt_override=None,
              compact: bool = False, exclusive: bool = False):
    """layers: list of dicts with 'q' and optionally 'k_swa', 'v_swa', 'gamma'.

    Returns a dict with o_full, lse_full, scores, idx, cnt and per-layer outputs.
    When idx_override/cnt_override are given, the sparse layers use those
    indices (used to check outputs independently of legitimate tie-band
    differences in the selection). ``exclusive`` selects the window-exclusive
    reading of the top-k candidates. With ``compact`` (and tile_ids) every
    output holds only the sampled tiles' rows, tile after tile, instead of
    full-size arrays with the other rows left NaN / 0.
    """
    compact = compact and tile_ids is not None
    o_full, lse_full = O.full_attention(q, k, v, cu_q, cu_kv, n_kv_heads, tiles_T=T,
                                        tile_ids=tile_ids, compact=compact)
    scores = O.importance_scores(q, k, lse_full, cu_q, cu_kv, n_kv_heads, T, B,
                                 tile_ids=tile_ids, compact=compact)
    idx, cnt = O.topk_select(scores, cu_q, cu_kv, T, B, topk, tile_ids=tile_ids, compact=compact, w=w,
                             exclusive=exclusive)
    use_idx = idx if idx_override is None else idx_override
    use_cnt = cnt if cnt_override is None else cnt_override
    outs = []
    rows = None if tile_ids is None else tile_rows(cu_q, cu_kv, T, tile_ids)
    for L in layers:
        o_sp, lse_sp = O.sparse_attention(L["q"], k, v, use_idx, use_cnt, cu_q, cu_kv, T, B, w,
                                          tile_ids=tile_ids, compact=compact)
        if swa_window > 0:
            o_swa, _ = O.swa_attention(L["q"], L["k_swa"], L["v_swa"], cu_q, cu_kv, swa_window,
                                       row_ids=rows, compact=compact)
            gamma = L["gamma"][rows] if compact else L["gamma"]
            o = O.gated_merge(gamma, o_sp, o_swa)
        else:
            o = o_sp
        outs.append({"o_sparse": o_sp, "lse_sparse": lse_sp, "o": o})
    return {"o_full": o_full, "lse_full": lse_full, "scores": scores, "idx": idx, "cnt": cnt,
            "layers": outs}
