"""GPU (libhs through its C ABI) against the fp64 oracle, element by element.

Whole-problem checks at sizes the oracle finishes in seconds (several tiles,
ragged tails, chunked prefill, GQA/MQA, both head dims), and sampled tiles of
the full-size HySparse block-level workload in the benchmark's launch
configuration.
"""
import numpy as np
import pytest
import torch

import oracle as O
from oracle.block import tile_rows
import workloads as W
from tests.parity import (GpuBlock, LazyF64, f64, assert_close_out, assert_close_lse, assert_scores_close,
                          assert_indices_match, FP8_MAX)

pytestmark = pytest.mark.gpu


class _Dequant:
    """float64 view of an FP8 KV cache: e4m3 codes times per-token scales."""

    def __init__(self, codes, scale):
        self.c, self.s = codes, scale
        self.shape = tuple(codes.shape)

    def __getitem__(self, idx):
        if isinstance(idx, tuple):
            idx = tuple(torch.from_numpy(i.astype(np.int64)).to(self.c.device) if isinstance(i, np.ndarray) else i
                        for i in idx)
        codes = self.c[idx].cpu().numpy()
        sc = self.s[idx[:2] if isinstance(idx, tuple) else idx].cpu().numpy()
        return O.dequant_fp8(codes, sc) if codes.ndim > sc.ndim else O.e4m3_to_f64(codes) * sc


class _Expand(_Dequant):
    """float64 values of the bf16 expansion of an FP8 cache, bf16_rn(scale * e4m3),
    formed by torch on the host (fp32 product, then bf16): the cache the FP8
    prefill path computes with."""

    def __getitem__(self, idx):
        if isinstance(idx, tuple):
            idx = tuple(torch.from_numpy(i.astype(np.int64)).to(self.c.device) if isinstance(i, np.ndarray) else i
                        for i in idx)
        codes = self.c[idx].cpu().view(torch.float8_e4m3fn).float()
        sc = self.s[idx[:2] if isinstance(idx, tuple) else idx].cpu().float()
        return f64((codes * sc.unsqueeze(-1)).to(torch.bfloat16))


def check_block(w, inp, res, tile_ids=None, fp8=False):
    """Compare every step of one hybrid block on the given tiles (None = all).

    The oracle runs in compact mode: only the sampled tiles' rows are computed
    and compared, so full-size workloads stay cheap on the host."""
    cu_q, cu_kv = w.cu_q(), w.cu_kv()
    T, B = w.q_tile, w.block
    dev = inp.q.device
    q, k, v = LazyF64(inp.q), LazyF64(inp.k), LazyF64(inp.v)
    kd, vd = (_Dequant(inp.k_fp8, inp.k_scale), _Dequant(inp.v_fp8, inp.v_scale)) if fp8 else (k, v)
    decode = T == 1 and all(n == 1 for n in w.new)
    # An FP8 cache in prefill is expanded once to bf16 and read by every layer:
    # the attention arithmetic is checked at the bf16 bars against the oracle
    # on that expansion (formed on the host), and the outputs end to end
    # against the oracle on the exact dequantised cache within the FP8 bar.
    # Decode reads the codes directly (exact fp16 expansion in the kernel).
    fp8_prefill = fp8 and not decode
    kf, vf = (_Expand(inp.k_fp8, inp.k_scale), _Expand(inp.v_fp8, inp.v_scale)) if fp8_prefill else (k, v)
    if fp8_prefill:
        kd, vd = kf, vf
    tiles = O.make_tiles(cu_q, cu_kv, T)
    tids = list(range(len(tiles))) if tile_ids is None else list(tile_ids)
    rows = tile_rows(cu_q, cu_kv, T, tids)
    rows_t = torch.tensor(rows, device=dev, dtype=torch.long)
    tids_t = torch.tensor(tids, device=dev, dtype=torch.long)
    # A1: full attention
    o_o, lse_o = O.full_attention(q, kf, vf, cu_q, cu_kv, w.n_kv_heads, tiles_T=T, tile_ids=tids, compact=True)
    assert_close_out(f64(res["o_full"][rows_t]), o_o, what="full o")
    assert_close_lse(f64(res["lse_full"][:, rows_t]), lse_o, what="full lse")
    if fp8_prefill:
        kx, vx = _Dequant(inp.k_fp8, inp.k_scale), _Dequant(inp.v_fp8, inp.v_scale)
        o_x, _ = O.full_attention(q, kx, vx, cu_q, cu_kv, w.n_kv_heads, tiles_T=T, tile_ids=tids, compact=True)
        assert_close_out(f64(res["o_full"][rows_t]), o_x, max_tol=FP8_MAX, mean_tol=1.0, what="full o, exact FP8")
    # A2: scores
    sc_o = O.importance_scores(q, kf, lse_o, cu_q, cu_kv, w.n_kv_heads, T, B, tile_ids=tids, compact=True)
    sc_g = f64(res["scores"][tids_t])
    assert_scores_close(sc_g, sc_o, range(len(tids)))
    # A3: top-k -- exact on the GPU's own scores, tie band against the oracle's
    idx_g = res["idx"][tids_t].cpu().numpy()[:, :, :w.topk]
    cnt_g = res["cnt"][tids_t].cpu().numpy()
    idx_x, cnt_x = O.topk_select(sc_g, cu_q, cu_kv, T, B, w.topk, tile_ids=tids, compact=True, w=w.window,
                                 exclusive=w.exclusive)
    assert (cnt_g == cnt_x).all(), "cnt of GPU scores differs"
    assert (idx_g == idx_x).all(), "top-k of GPU scores differs"
    idx_o, cnt_o = O.topk_select(sc_o, cu_q, cu_kv, T, B, w.topk, tile_ids=tids, compact=True, w=w.window,
                                 exclusive=w.exclusive)
    assert_indices_match(idx_g, cnt_g, sc_o, idx_o, cnt_o, range(len(tids)), max(w.topk, 1))
    # A4 / A5 / A6: sparse layers, fed the GPU's (checked) indices
    for li, (L, Lg) in enumerate(zip(inp.layers, res["layers"])):
        ql = LazyF64(L.q)
        o_sp, lse_sp = O.sparse_attention(ql, kd, vd, idx_g, cnt_g, cu_q, cu_kv, T, B, w.window, tile_ids=tids,
                                          compact=True)
        o_sp_g = f64(Lg["o_sparse"][rows_t])
        assert_close_out(o_sp_g, o_sp, what=f"layer {li} sparse o")
        assert_close_lse(f64(Lg["lse_sparse"][:, rows_t]), lse_sp, what=f"layer {li} sparse lse")
        if fp8 and decode:  # and against the bf16-KV oracle within the FP8 bound
            # (decode rows average over k + w keys; prefill rows near a sequence
            # start see one or two keys, whose e4m3 error, up to 2^-4 relative,
            # no average hides: there the bound is checked against the exact
            # dequantised cache below)
            o_bf, _ = O.sparse_attention(ql, k, v, idx_g, cnt_g, cu_q, cu_kv, T, B, w.window, tile_ids=tids,
                                         compact=True)
            assert_close_out(o_sp_g, o_bf, max_tol=FP8_MAX, mean_tol=1.0, what=f"layer {li} fp8 vs bf16 KV")
        if fp8_prefill:  # and against the exact dequantised cache within the FP8 bound
            o_x, _ = O.sparse_attention(ql, _Dequant(inp.k_fp8, inp.k_scale), _Dequant(inp.v_fp8, inp.v_scale),
                                        idx_g, cnt_g, cu_q, cu_kv, T, B, w.window, tile_ids=tids, compact=True)
            assert_close_out(o_sp_g, o_x, max_tol=FP8_MAX, mean_tol=1.0, what=f"layer {li} exact FP8")
        if w.swa_window > 0:
            o_swa, _ = O.swa_attention(ql, LazyF64(L.k_swa), LazyF64(L.v_swa), cu_q, cu_kv, w.swa_window,
                                       row_ids=rows, compact=True)
            gamma = f64(L.gamma[rows_t])
            # gate applied to the GPU's bf16 sparse output (the call's actual input)
            o_gate = O.gated_merge(gamma, o_sp_g, o_swa)
            o_l = f64(Lg["o"][rows_t])
            assert_close_out(o_l, o_gate, what=f"layer {li} gated o")
            # and the whole chain against the oracle's own sparse output
            assert_close_out(o_l, O.gated_merge(gamma, o_sp, o_swa), what=f"layer {li} chain o")


def check_fused_topk(w, blk, inp, res, fp8=False):
    """Token-level prefill: hs_full_attn_select_topk (the top-k taken inside the
    score pass) returns exactly the o, lse, idx and cnt of the two calls the
    block ran (full layer, then hs_topk_select on the stored scores), whole
    arrays including the -1 padding."""
    import hybrid_sparse_attention_tma_b200 as hs
    if w.block != 1 or blk.block.decode:
        return
    k, v = inp.k, inp.v
    if fp8:  # the block expanded the FP8 cache once; the full layer read that
        k, v = blk.block._bufs["k_deq"], blk.block._bufs["v_deq"]
    ws = hs.Workspace("cuda")
    o, lse, idx, cnt = hs.full_attn_select_topk(blk.vl, blk.sel, inp.q, k, v, ws=ws)
    hs.check_error(ws)
    assert torch.equal(cnt, res["cnt"]), "fused top-k: cnt differs from the two-call path"
    assert torch.equal(idx, res["idx"]), "fused top-k: idx differs from the two-call path"
    assert torch.equal(o.view(torch.int16), res["o_full"].view(torch.int16))
    assert torch.equal(lse.view(torch.int32), res["lse_full"].view(torch.int32))


def run_and_check(w, seed=None, tile_ids=None, fp8=False, fused=True):
    import sys, time
    t0 = time.time()
    inp = W.make_block_inputs(w, device="cuda", seed=seed)
    torch.cuda.synchronize()
    t1 = time.time()
    blk = GpuBlock(w, inp, fused=fused)
    res = blk.run(fp8=fp8)
    torch.cuda.synchronize()
    t2 = time.time()
    check_block(w, inp, res, tile_ids, fp8=fp8)
    check_fused_topk(w, blk, inp, res, fp8=fp8)
    print(f"[{w.name}] inputs {t1 - t0:.1f}s gpu {t2 - t1:.2f}s oracle check {time.time() - t2:.1f}s",
          file=sys.stderr, flush=True)
    return inp, res


def test_tiny_config_whole():
    run_and_check(W.WORKLOADS["tiny"])


VARIANTS = {
    # chunked prefill, ragged tails, GQA group 4, d=128, 64-token blocks, no window
    "gqa4_d128_b64_w0": W.Workload("v1", ctx=(0, 300, 37), new=(200, 333, 130), n_q_heads=8, n_kv_heads=2,
                                   head_dim=128, q_tile=64, block=64, topk=3, window=0, n_sparse=1),
    # MQA with 16 heads, window 128, blocks of 16, tile 16
    "mqa16_d128_b16_w128": W.Workload("v2", ctx=(0, 257), new=(300, 77), n_q_heads=16, n_kv_heads=1,
                                      head_dim=128, q_tile=16, block=16, topk=8, window=128, n_sparse=1),
    # MHA (G=1), d=64, block 32, window 16
    "mha_d64_b32": W.Workload("v3", ctx=(5,), new=(259,), n_q_heads=2, n_kv_heads=2, head_dim=64,
                              q_tile=32, block=32, topk=2, window=16, n_sparse=1),
    # k >= all candidates: sparse must equal full attention
    "k_all": W.Workload("v4", ctx=(0,), new=(256,), n_q_heads=4, n_kv_heads=1, head_dim=64, q_tile=64,
                        block=16, topk=64, window=0, n_sparse=1),
    # k = 0 with a window: sparse = window-only attention
    "k0_window": W.Workload("v5", ctx=(0,), new=(200,), n_q_heads=4, n_kv_heads=1, head_dim=64, q_tile=16,
                            block=16, topk=0, window=24, n_sparse=1),
    # G = 128 (two queries per M tile)
    "g128": W.Workload("v6", ctx=(60,), new=(9,), n_q_heads=128, n_kv_heads=1, head_dim=128, q_tile=4,
                       block=8, topk=4, window=8, n_sparse=1),
    # token level (B = 1): MQA 32 heads, window 32, chunked + ragged
    "tok_mqa32": W.Workload("v8", ctx=(0, 700), new=(300, 180), n_q_heads=32, n_kv_heads=1, head_dim=128,
                            q_tile=16, block=1, topk=96, window=32, n_sparse=1, needle_rate=0.02),
    # token level, GQA 4, d = 64, k larger than some tiles' candidates
    "tok_gqa4_d64": W.Workload("v9", ctx=(40,), new=(400,), n_q_heads=8, n_kv_heads=2, head_dim=64, q_tile=64,
                               block=1, topk=200, window=16, n_sparse=1),
    # SWA + gate branch at small size
    "swa_gate": W.Workload("v7", ctx=(0, 100), new=(300, 200), n_q_heads=8, n_kv_heads=2, head_dim=128,
                           q_tile=64, block=64, topk=2, window=0, n_sparse=2, swa_window=128),
    # a sequence with no new tokens inside the batch, fused layer with 16-token blocks
    "empty_seq": W.Workload("v10", ctx=(0, 90, 40), new=(150, 0, 70), n_q_heads=4, n_kv_heads=1, head_dim=64,
                            q_tile=16, block=16, topk=4, window=8, n_sparse=1, swa_window=32),
    # window-exclusive top-k (k global tokens + the latest w), token level, chunked + ragged
    "tok_exclusive": W.Workload("v12", ctx=(0, 500), new=(300, 150), n_q_heads=32, n_kv_heads=1, head_dim=128,
                                q_tile=16, block=1, topk=96, window=32, n_sparse=1, needle_rate=0.02, exclusive=True),
    # window-exclusive top-k at block level, GQA
    "blk_exclusive": W.Workload("v13", ctx=(64, 0), new=(260, 200), n_q_heads=8, n_kv_heads=2, head_dim=64,
                                q_tile=32, block=16, topk=4, window=24, n_sparse=1, exclusive=True),
    # token level with G = 128 (two queries per 256-row score chunk) and with G = 1 (MHA, d = 64: a
    # 64-query tile fills a quarter of a score chunk)
    "tok_g128": W.Workload("v14", ctx=(37,), new=(50,), n_q_heads=128, n_kv_heads=1, head_dim=128, q_tile=4,
                           block=1, topk=24, window=8, n_sparse=1),
    "tok_mha_d64": W.Workload("v15", ctx=(0, 130), new=(300, 45), n_q_heads=2, n_kv_heads=2, head_dim=64,
                              q_tile=64, block=1, topk=40, window=16, n_sparse=1),
    # token-level selection with the window branch and gate fused in (one launch per layer)
    "swa_tok": W.Workload("v11", ctx=(0, 300), new=(260, 90), n_q_heads=16, n_kv_heads=1, head_dim=128,
                          q_tile=16, block=1, topk=64, window=8, n_sparse=1, swa_window=32, needle_rate=0.02),
}


@pytest.mark.parametrize("name", list(VARIANTS))
def test_variant_whole(name):
    run_and_check(VARIANTS[name], seed=7)


# The kernels are checked at the bf16 bars against the oracle on the expanded
# cache and, end to end, within the FP8 bar against the exact dequantised cache.
FP8_PREFILL = {
    # token level, MQA, chunked + ragged, forced window
    "fp8_tok_mqa": VARIANTS["tok_mqa32"].with_(needle_rate=0.0),
    # block level, GQA, own-cache window branch + gate fused in
    "fp8_swa_gate": VARIANTS["swa_gate"],
    # window-exclusive token level
    "fp8_tok_exclusive": VARIANTS["tok_exclusive"].with_(needle_rate=0.0),
}


@pytest.mark.parametrize("name", list(FP8_PREFILL))
def test_fp8_kv_prefill_whole(name):
    """Prefill over an FP8-e4m3 KV cache (per-token scales): the block expands
    the cache once and every layer reads it; checked against the oracle on the
    dequantised cache, and against the bf16-KV oracle within the FP8 bound."""
    w = FP8_PREFILL[name].with_(fp8_kv=True)
    run_and_check(w, seed=7, fp8=True)


def test_fp8_kv_prefill_full_size_sampled_tiles():
    """HySparse2 token-level prefill at full size over an FP8 KV cache,
    sampled tiles (first, middle, last)."""
    w = W.WORKLOADS["hys2_prefill"].with_(fp8_kv=True, n_sparse=2, needle_rate=0.0)
    n_t = w.n_tiles()
    run_and_check(w, tile_ids=[0, n_t // 2, n_t - 1], fp8=True)


@pytest.mark.parametrize("name", ["tok_mqa32", "tok_gqa4_d64", "tok_exclusive"])
def test_gathered_rows_and_layer_match_the_per_tile_gather(name):
    """Token level: hs_gather_selected_kv copies exactly the selected rows of
    every (tile, KV head), zero past cnt (against a host gather), and the
    sparse layer reading them equals the layer that gathers each tile with
    tile::gather4, bit for bit (o and lse). The block runner uses the gathered
    layer, so the oracle checks of the token-level variants cover it."""
    import hybrid_sparse_attention_tma_b200 as hs
    w = VARIANTS[name]
    inp = W.make_block_inputs(w, device="cuda", seed=13)
    blk = GpuBlock(w, inp)
    res = blk.run()
    idx, cnt = res["idx"], res["cnt"]
    kg, vg = hs.gather_selected_kv(blk.vl, blk.sel, inp.k, inp.v, idx, cnt)
    L0 = inp.layers[0]
    o_a, lse_a = hs.sparse_attn_prefill(blk.vl, blk.sel, L0.q, inp.k, inp.v, idx, cnt)
    o_b, lse_b = hs.sparse_attn_prefill(blk.vl, blk.sel, L0.q, inp.k, inp.v, idx, cnt, kg=kg, vg=vg)
    torch.cuda.synchronize()
    assert torch.equal(o_a.view(torch.int16), o_b.view(torch.int16))
    assert torch.equal(lse_a.view(torch.int32), lse_b.view(torch.int32))
    # host gather of the selected rows
    cu_q, cu_kv, T = w.cu_q(), w.cu_kv(), w.q_tile
    k_h, v_h, idx_h, cnt_h = inp.k.cpu(), inp.v.cpu(), idx.cpu(), cnt.cpu()
    kg_ref = torch.zeros(tuple(kg.shape), dtype=torch.bfloat16)
    vg_ref = torch.zeros(tuple(vg.shape), dtype=torch.bfloat16)
    tile = 0
    for b in range(len(cu_q) - 1):
        n_b = cu_q[b + 1] - cu_q[b]
        for _ in range((n_b + T - 1) // T):
            for g in range(w.n_kv_heads):
                c = int(cnt_h[tile, g])
                rows = cu_kv[b] + idx_h[tile, g, :c].long()
                kg_ref[tile, g, :c] = k_h[rows, g]
                vg_ref[tile, g, :c] = v_h[rows, g]
            tile += 1
    assert tile == kg.shape[0]
    assert torch.equal(kg.cpu().view(torch.int16), kg_ref.view(torch.int16))
    assert torch.equal(vg.cpu().view(torch.int16), vg_ref.view(torch.int16))


@pytest.mark.parametrize("name", ["tok_mqa32", "swa_gate", "dec_block_swa"])
def test_forward_from_host_equals_forward(name):
    """HybridBlock.forward_from_host (inputs in pinned host memory, each layer's
    inputs streamed in under the earlier layers' compute) writes exactly what
    forward() writes on device inputs, with a slot per layer and with two slots
    (three sparse layers, so a slot is refilled)."""
    from hybrid_sparse_attention_tma_b200.block import SparseLayerIn
    w = (VARIANTS.get(name) or DECODE[name]).with_(n_sparse=3)
    inp = W.make_block_inputs(w, device="cuda", seed=21)
    blk = GpuBlock(w, inp)
    a = blk.run()
    ref = {"o_full": a["o_full"].clone(), "idx": a["idx"].clone(),
           "o": [L["o"].clone() for L in a["layers"]]}
    pin = (lambda t: None if t is None else t.cpu().pin_memory())
    hl = [SparseLayerIn(pin(L.q), pin(L.k_swa), pin(L.v_swa), pin(L.gamma)) for L in blk.layers]
    for slots in (None, 2):  # a slot per layer; two slots, refilled
        b = blk.block.forward_from_host(pin(inp.q), pin(inp.k), pin(inp.v), hl, slots=slots)
        torch.cuda.synchronize()
        assert torch.equal(ref["o_full"], b["o_full"]) and torch.equal(ref["idx"], b["idx"])
        assert torch.equal(ref["o"][-1], b["layers"][-1]["o"])
        assert torch.equal(ref["o"][-2], b["layers"][-2]["o"])


FUSED_TOPK_CASES = ["random", "dup_rows", "all_equal", "exclusive", "k_over_n", "k0", "d64_gqa", "block16",
                    "decode"]


@pytest.mark.parametrize("case", FUSED_TOPK_CASES)
def test_fused_topk_equals_two_calls_on_ties_and_edges(case):
    """hs_full_attn_select_topk against hs_full_attn_select + hs_topk_select on
    inputs built for the selection's hard cases: K rows repeating with period
    37 (equal scores for every key the same queries see: ties broken toward
    the lower index), all-zero K (every visible key tied), the
    window-exclusive reading, k above every tile's candidates, k = 0, d = 64
    with GQA, plus the shapes that run the two calls inside (block level,
    decode). o, lse, cnt and the kept indices must match exactly."""
    import hybrid_sparse_attention_tma_b200 as hs
    g = torch.Generator().manual_seed(5)
    Hq, Hkv, d, T, B = 16, 1, 128, 16, 1
    cu_q, cu_kv = [0, 300, 480, 481], [0, 1000, 1180, 1700]  # chunked, fresh, one query
    if case == "d64_gqa":
        Hq, Hkv, d = 8, 2, 64
    if case == "block16":
        B = 16
    if case == "decode":
        T, cu_q = 1, [0, 1, 2, 3]
    Tq, Tkv = cu_q[-1], cu_kv[-1]
    q = torch.randn(Tq, Hq, d, generator=g).to(torch.bfloat16)
    k = torch.randn(Tkv, Hkv, d, generator=g).to(torch.bfloat16)
    v = torch.randn(Tkv, Hkv, d, generator=g).to(torch.bfloat16)
    if case == "dup_rows":
        k = k[torch.arange(Tkv) % 37]
    if case == "all_equal":
        k = torch.zeros_like(k)
    topk = {"k_over_n": 2000, "k0": 0}.get(case, 96)
    window = 32
    vl = hs.Varlen(cu_q, cu_kv, Hq, Hkv, d, device="cuda")
    sel = hs.Sel(T, B, topk, window, case == "exclusive")
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    ws = hs.Workspace("cuda")
    o1, lse1, sc = hs.full_attn_select(vl, sel, q, k, v, ws=ws)
    idx1, cnt1 = hs.topk_select(vl, sel, sc, ws=ws)
    o2, lse2, idx2, cnt2 = hs.full_attn_select_topk(vl, sel, q, k, v, ws=ws)
    hs.check_error(ws)
    assert torch.equal(cnt1, cnt2)
    if topk > 0:
        assert torch.equal(idx1, idx2)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(lse1.view(torch.int32), lse2.view(torch.int32))
    if case == "all_equal" and B == 1:
        # every candidate of a plane whose first query sees it is tied: the kept
        # set of each tile starts at index 0
        c = cnt2.cpu()
        assert (idx2.cpu()[:, 0, 0][c[:, 0] > 0] == 0).all()


@pytest.mark.parametrize("name", ["tok_mqa32", "swa_tok"])
def test_block_with_fused_topk_equals_two_call_block(name):
    """The block runner with fuse_topk (top-k inside the score pass) writes
    exactly what the two-call block writes, every layer."""
    from hybrid_sparse_attention_tma_b200.block import HybridBlock
    w = VARIANTS[name].with_(n_sparse=2)
    inp = W.make_block_inputs(w, device="cuda", seed=17)
    a = GpuBlock(w, inp).run()
    ref = {"idx": a["idx"].clone(), "cnt": a["cnt"].clone(), "o": [L["o"].clone() for L in a["layers"]]}
    fb = GpuBlock(w, inp, fuse_topk=True)
    assert fb.block.fuse_topk
    b = fb.run()
    torch.cuda.synchronize()
    assert b["scores"] is None
    assert torch.equal(ref["cnt"], b["cnt"]) and torch.equal(ref["idx"], b["idx"])
    for x, y in zip(ref["o"], b["layers"]):
        assert torch.equal(x.view(torch.int16), y["o"].view(torch.int16))


def test_swa_gate_two_call_path():
    """The unfused layer (hs_sparse_attn_prefill then hs_swa_gated) against the oracle."""
    run_and_check(VARIANTS["swa_gate"], seed=7, fused=False)


def test_fused_layer_without_intermediates_writes_the_same_output():
    """o_sparse / lse_sparse are optional outputs of the fused layer: leaving
    them out changes no bit of o."""
    w = VARIANTS["swa_gate"]
    inp = W.make_block_inputs(w, device="cuda", seed=9)
    blk = GpuBlock(w, inp)
    a = [L["o"].clone() for L in blk.run()["layers"]]
    b = blk.run(intermediates=False)["layers"]
    for x, y in zip(a, b):
        assert y["o_sparse"] is None and y["lse_sparse"] is None
        assert torch.equal(x, y["o"])


def test_k_all_equals_full_attention_on_gpu():
    w = VARIANTS["k_all"]
    inp = W.make_block_inputs(w, device="cuda", seed=3)
    import hybrid_sparse_attention_tma_b200 as hs
    blk = GpuBlock(w, inp)
    res = blk.run()
    o_f, lse_f, _ = hs.full_attn_select(blk.vl, blk.sel, inp.layers[0].q, inp.k, inp.v)
    torch.cuda.synchronize()
    assert_close_out(f64(res["layers"][0]["o_sparse"]), f64(o_f), what="k>=all vs full")
    assert_close_lse(f64(res["layers"][0]["lse_sparse"]), f64(lse_f), what="k>=all lse vs full")


def test_hys_block_full_size_sampled_tiles():
    """HySparse block-level prefill at full size (32768 tokens, 32/8 heads,
    d=128, B=64, k=16, SWA 128 + gate), 3 sparse layers, checked on sampled
    tiles including the first and the last."""
    w = W.WORKLOADS["hys_block"]
    n_t = w.n_tiles()
    rng = np.random.default_rng(11)
    tiles = sorted({0, n_t - 1, *rng.choice(n_t, size=2, replace=False).tolist()})
    run_and_check(w, tile_ids=tiles)


def test_hys2_token_full_size_sampled_tiles():
    """HySparse2 token-level prefill at full size (65536 tokens, 64/1 heads,
    d=128, top-1024 + forced 128, tile 64), 11 sparse layers, sampled tiles."""
    w = W.WORKLOADS["hys2_prefill"]
    n_t = w.n_tiles()
    rng = np.random.default_rng(12)
    tiles = sorted({0, n_t - 1, *rng.choice(n_t, size=1, replace=False).tolist()})
    run_and_check(w, tile_ids=tiles)


def test_hys2_token_full_size_exclusive_sampled_tiles():
    """HySparse2 token-level prefill at full size with the window-exclusive
    reading (top-1024 global tokens + the latest 128), sampled tiles."""
    w = W.WORKLOADS["hys2_prefill"].with_(exclusive=True, n_sparse=2)
    n_t = w.n_tiles()
    run_and_check(w, tile_ids=[0, n_t // 3, n_t - 1])


def test_agentic_chunked_full_size_sampled_tiles():
    """Agentic ragged chunked prefill at full size (contexts 262144/131072/65536/
    16384 + chunks 8192/4096/8192/2048, 64/1 heads, top-1024 + forced 128),
    sampled tiles from every sequence."""
    w = W.WORKLOADS["agentic"]
    tiles = O.make_tiles(w.cu_q(), w.cu_kv(), w.q_tile)
    first = {}
    for t in tiles:
        first.setdefault(t.seq, []).append(t.index)
    pick = sorted({first[0][-1], first[1][0], first[2][len(first[2]) // 2], first[3][-1]})
    run_and_check(w, tile_ids=pick)


DECODE = {
    # MQA 64 heads, ragged contexts (one not a multiple of anything), k = 64, w = 32
    "dec_mqa": W.Workload("d1", ctx=(300, 1000, 128, 2000, 63), new=(1,) * 5, n_q_heads=64, n_kv_heads=1,
                          head_dim=128, q_tile=1, block=1, topk=64, window=32, n_sparse=2),
    # GQA group 8 (only 8 of the 64 MMA rows valid), several KV heads
    "dec_gqa8": W.Workload("d2", ctx=(700, 90), new=(1, 1), n_q_heads=32, n_kv_heads=4, head_dim=128,
                           q_tile=1, block=1, topk=40, window=16, n_sparse=1),
    # window-exclusive decode: 1024-style global tokens plus the latest w, disjoint
    "dec_exclusive": W.Workload("d4", ctx=(900, 130, 2000), new=(1, 1, 1), n_q_heads=64, n_kv_heads=1,
                                head_dim=128, q_tile=1, block=1, topk=80, window=48, n_sparse=1, exclusive=True),
    # k = 0: the sparse layer sees only the forced window (one context shorter than the window)
    "dec_window_only": W.Workload("d3", ctx=(200, 45), new=(1, 1), n_q_heads=64, n_kv_heads=1, head_dim=128,
                                  q_tile=1, block=1, topk=0, window=48, n_sparse=1),
    # HySparse layer shape at decode time: 64-token blocks, top-4, no forced window,
    # own sliding-window branch over a 128-slot ring + sigmoid gate; ragged
    # contexts (one shorter than the window, one a multiple of the block)
    "dec_block_swa": W.Workload("d5", ctx=(300, 1000, 63, 2047), new=(1,) * 4, n_q_heads=16, n_kv_heads=4,
                                head_dim=128, q_tile=1, block=64, topk=4, window=0, n_sparse=2, swa_window=128),
    # block-level decode with a forced window (16-token blocks), GQA 4
    "dec_block_window": W.Workload("d6", ctx=(500, 77), new=(1, 1), n_q_heads=8, n_kv_heads=2, head_dim=128,
                                   q_tile=1, block=16, topk=6, window=24, n_sparse=1),
}


@pytest.mark.parametrize("name", list(DECODE))
@pytest.mark.parametrize("fp8", [False, True])
def test_decode_whole(name, fp8):
    w = DECODE[name].with_(fp8_kv=True)
    run_and_check(w, seed=5, fp8=fp8)


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_split_counts_agree_with_the_oracle(fp8):
    """Every way of cutting a unit's slots into key ranges (one range, the
    automatic count, one tile per range, more ranges than tiles) gives the
    oracle's sparse-layer output; the ranges are merged by log-sum-exp."""
    import hybrid_sparse_attention_tma_b200 as hs
    w = W.Workload("dsplit", ctx=(1500, 700, 300), new=(1, 1, 1), n_q_heads=64, n_kv_heads=1, head_dim=128,
                   q_tile=1, block=1, topk=500, window=40, n_sparse=1, fp8_kv=True)
    inp = W.make_block_inputs(w, device="cuda", seed=17)
    blk = GpuBlock(w, inp)
    res = blk.run(fp8=fp8)
    torch.cuda.synchronize()
    idx, cnt = res["idx"], res["cnt"]
    L0 = inp.layers[0]
    kd, vd = (_Dequant(inp.k_fp8, inp.k_scale), _Dequant(inp.v_fp8, inp.v_scale)) if fp8 else (LazyF64(inp.k),
                                                                                                   LazyF64(inp.v))
    cu_q, cu_kv = w.cu_q(), w.cu_kv()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    o_ref, lse_ref = O.sparse_attention(LazyF64(L0.q), kd, vd, idx_h, cnt_h, cu_q, cu_kv, 1, 1, w.window)
    tiles = (w.topk + w.window + 127) // 128
    for split in [1, 2, tiles, tiles + 5]:
        if fp8:
            o, lse = hs.sparse_attn_decode(blk.vl, blk.sel, L0.q, inp.k_fp8, inp.v_fp8, idx, cnt, inp.k_scale,
                                           inp.v_scale, hs.HS_KV_FP8_E4M3, split_k=split)
        else:
            o, lse = hs.sparse_attn_decode(blk.vl, blk.sel, L0.q, inp.k, inp.v, idx, cnt, split_k=split)
        torch.cuda.synchronize()
        assert_close_out(f64(o), o_ref, what=f"split {split} o")
        assert_close_lse(f64(lse), lse_ref, what=f"split {split} lse")


@pytest.mark.parametrize("fp8", [False, True])
def test_decode_full_size_sampled_sequences(fp8):
    """Token-level decode at full size: 64 sequences x 131072 cached tokens,
    64/1 heads, top-1024 + forced 128, bf16 and FP8-e4m3 KV (per-token scales)."""
    w = W.WORKLOADS["decode"].with_(fp8_kv=True, n_sparse=2)
    run_and_check(w, tile_ids=[0, 17, 63], fp8=fp8)


def test_bounded_wait_timeout_reports_and_context_survives():
    import ctypes
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200 import _lib as L
    ws = hs.Workspace("cuda")
    buf = ws.get(4096)
    lib = L.load()
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.hs_debug_wait_timeout(ctypes.c_void_p(buf.data_ptr()), buf.numel(), 2_000_000, s) == L.HS_OK
    with pytest.raises(hs.HsError) as e:
        hs.check_error(ws)
    assert e.value.status == L.HS_ERR_TIMEOUT
    hs.check_error(ws)  # cleared
    run_and_check(VARIANTS["k0_window"], seed=1)


def test_empty_batch_is_a_no_op():
    """Every call accepts a batch without new tokens (empty tensors, null data
    pointers) and returns without launching; the block runner passes through.
    The decode entry point likewise accepts a batch of no sequences."""
    w = W.Workload("e0", ctx=(64, 100), new=(0, 0), n_q_heads=8, n_kv_heads=2, head_dim=128, q_tile=64, block=64,
                   topk=2, window=0, n_sparse=2, swa_window=128)
    inp = W.make_block_inputs(w, device="cuda", seed=1)
    assert inp.q.shape[0] == 0
    res = GpuBlock(w, inp).run()
    torch.cuda.synchronize()
    assert res["o_full"].shape[0] == 0 and res["scores"].shape[0] == 0
    for L in res["layers"]:
        assert L["o"].shape[0] == 0
