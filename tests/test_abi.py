"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from hybrid_sparse_attention_tma_b200 import build, _lib
    build.build()
    return _lib.load()


def header_functions():
    with open(os.path.join(ROOT, "include", "hs.h")) as f:
        src = f.read()
    return sorted(set(re.findall(r"HS_API\s+[\w\s\*]+?\b(hs_\w+)\s*\(", src)))


def test_header_declares_the_five_calls():
    names = header_functions()
    for n in ["hs_full_attn_select", "hs_topk_select", "hs_sparse_attn_prefill", "hs_sparse_attn_decode",
              "hs_swa_gated"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from hybrid_sparse_attention_tma_b200 import _lib
    for n in header_functions():
        assert hasattr(lib, n), n
    assert sorted(_lib.EXPORTS) == header_functions()


def test_status_strings(lib):
    for s in range(6):
        assert lib.hs_status_string(s)


def _varlen(cu_q, cu_kv, hq=4, hkv=1, d=64):
    from hybrid_sparse_attention_tma_b200 import _lib as L
    cq = (ctypes.c_int32 * len(cu_q))(*cu_q)
    ckv = (ctypes.c_int32 * len(cu_kv))(*cu_kv)
    vl = L.HsVarlen(len(cu_q) - 1, hq, hkv, d, 16, 16, cq, ckv, 0.0)
    vl._keep = (cq, ckv)
    return vl


def test_workspace_size_and_validation(lib):
    from hybrid_sparse_attention_tma_b200 import _lib as L
    vl = _varlen([0, 512], [0, 512])
    sel = L.HsSel(16, 16, 8, 32)
    n = lib.hs_workspace_size(L.HS_OP_FULL_ATTN_SELECT, ctypes.byref(vl), ctypes.byref(sel))
    assert n >= 256 and n % 256 == 0
    assert lib.hs_workspace_size(L.HS_OP_TOPK_SELECT, ctypes.byref(vl), ctypes.byref(sel)) >= 256
    bad = _varlen([0, 512], [0, 100])  # fewer keys than queries
    assert lib.hs_workspace_size(L.HS_OP_FULL_ATTN_SELECT, ctypes.byref(bad), ctypes.byref(sel)) == 0


def _call_full(lib, vl, sel, ptr=16, ws=16, ws_bytes=1 << 30):
    return lib.hs_full_attn_select(ctypes.byref(vl) if vl is not None else None,
                                   ctypes.byref(sel) if sel is not None else None,
                                   ptr, ptr, ptr, ptr, ptr, ptr, ws, ws_bytes, None)


def test_host_validation_errors(lib):
    from hybrid_sparse_attention_tma_b200 import _lib as L
    vl = _varlen([0, 512], [0, 512])
    sel = L.HsSel(16, 16, 8, 32)
    assert _call_full(lib, None, sel) == L.HS_ERR_INVALID_ARG
    assert _call_full(lib, vl, None) == L.HS_ERR_INVALID_ARG
    assert _call_full(lib, vl, sel, ptr=None) == L.HS_ERR_INVALID_ARG
    assert _call_full(lib, vl, sel, ptr=18) == L.HS_ERR_INVALID_ARG          # misaligned
    assert _call_full(lib, vl, sel, ws=None) == L.HS_ERR_WORKSPACE
    assert _call_full(lib, vl, sel, ws_bytes=8) == L.HS_ERR_WORKSPACE
    assert _call_full(lib, _varlen([0, 512], [0, 512], d=96), sel) == L.HS_ERR_UNSUPPORTED
    assert _call_full(lib, _varlen([0, 512], [0, 512], hq=6, hkv=4), sel) == L.HS_ERR_INVALID_ARG
    assert _call_full(lib, vl, L.HsSel(16, 24, 8, 32)) == L.HS_ERR_UNSUPPORTED  # block not a power of 2
    assert _call_full(lib, vl, L.HsSel(16, 16, 5000, 32)) == L.HS_ERR_UNSUPPORTED
    assert _call_full(lib, vl, L.HsSel(0, 16, 8, 32)) == L.HS_ERR_INVALID_ARG
    assert _call_full(lib, _varlen([0, 600], [0, 512]), sel) == L.HS_ERR_INVALID_ARG
    assert lib.hs_swa_gated(ctypes.byref(vl), 0, 16, 16, 16, 16, 16, 16, 16, 1 << 20, None) == L.HS_ERR_INVALID_ARG
    assert lib.hs_topk_select(ctypes.byref(vl), ctypes.byref(sel), None, 16, 16, 16, 1 << 20, None) == L.HS_ERR_INVALID_ARG
    # fused sparse layer: window, own cache and gate are required, pointers 16-byte aligned
    fused = lambda win, ks, osp: lib.hs_sparse_swa_gated_prefill(
        ctypes.byref(vl), ctypes.byref(sel), 16, 16, 16, 16, 16, win, ks, 16, 16, 16, osp, None, 16, 1 << 20, None)
    assert fused(0, 16, None) == L.HS_ERR_INVALID_ARG
    assert fused(128, None, None) == L.HS_ERR_INVALID_ARG
    assert fused(128, 16, 24) == L.HS_ERR_INVALID_ARG
    assert lib.hs_debug_wait_timeout(None, 0, 1000, None) == L.HS_ERR_WORKSPACE
    assert lib.hs_debug_wait_timeout(16, 1 << 20, 0, None) == L.HS_ERR_INVALID_ARG
    # FP8 expansion: empty is a no-op; bad sizes / pointers are rejected before launch
    assert lib.hs_kv_dequantize(None, None, 0, 128, None, None) == L.HS_OK
    assert lib.hs_kv_dequantize(16, 16, 4, 120, 16, None) == L.HS_ERR_INVALID_ARG  # head_dim % 16
    assert lib.hs_kv_dequantize(None, 16, 4, 128, 16, None) == L.HS_ERR_INVALID_ARG
    assert lib.hs_kv_dequantize(16, 18, 4, 128, 16, None) == L.HS_ERR_INVALID_ARG  # misaligned scale
    assert lib.hs_kv_dequantize(16, 16, -1, 128, 16, None) == L.HS_ERR_INVALID_ARG
    # rows gathered once per block: token level only; topk = 0 is a no-op; null
    # or misaligned buffers are rejected before launch, also by the layer reading them
    tok = L.HsSel(16, 1, 8, 32)
    gath = lambda s_, kg, vg: lib.hs_gather_selected_kv(ctypes.byref(vl), ctypes.byref(s_), 16, 16, 16, 16, kg, vg,
                                                        None)
    assert gath(sel, 16, 16) == L.HS_ERR_INVALID_ARG       # block 16
    assert gath(tok, None, 16) == L.HS_ERR_INVALID_ARG
    assert gath(tok, 16, 24) == L.HS_ERR_INVALID_ARG       # misaligned
    assert gath(L.HsSel(16, 1, 0, 32), None, None) == L.HS_OK
    layer = lambda s_, kg: lib.hs_sparse_attn_prefill_gathered(ctypes.byref(vl), ctypes.byref(s_), 16, 16, 16, kg,
                                                               16, 16, 16, 16, 16, 16, 1 << 20, None)
    assert layer(sel, 16) == L.HS_ERR_INVALID_ARG          # block 16
    assert layer(tok, None) == L.HS_ERR_INVALID_ARG
    assert layer(tok, 40) == L.HS_ERR_INVALID_ARG          # misaligned
    # SWA ring: ring length >= 1, pointers 16-byte aligned; the decode branch needs
    # one new token per sequence and 1 <= window <= ring length (window <= 128)
    assert lib.hs_swa_ring_write(ctypes.byref(vl), 0, 16, 16, 16, 16, None) == L.HS_ERR_INVALID_ARG
    assert lib.hs_swa_ring_write(ctypes.byref(vl), 8, 16, 24, 16, 16, None) == L.HS_ERR_INVALID_ARG
    dec = _varlen([0, 1, 2], [0, 300, 600])
    swad = lambda vl_, win, ring, gam: lib.hs_swa_gated_decode(ctypes.byref(vl_), win, ring, 16, 16, 16, gam, 16,
                                                                16, None)
    assert swad(vl, 128, 128, 16) == L.HS_ERR_INVALID_ARG       # 512 new tokens in one sequence
    assert swad(dec, 0, 128, 16) == L.HS_ERR_INVALID_ARG
    assert swad(dec, 128, 64, 16) == L.HS_ERR_INVALID_ARG       # ring shorter than the window
    assert swad(dec, 256, 256, 16) == L.HS_ERR_UNSUPPORTED
    assert swad(dec, 128, 128, None) == L.HS_ERR_INVALID_ARG
    assert swad(dec, 128, 128, 18) == L.HS_ERR_INVALID_ARG      # misaligned gate
    # full layer + fused top-k: idx and cnt are required; the full layer's checks apply
    ftk = lambda vl_, s_, idx, cnt, ptr=16, ws_bytes=1 << 30: lib.hs_full_attn_select_topk(
        ctypes.byref(vl_) if vl_ is not None else None, ctypes.byref(s_), ptr, ptr, ptr, ptr, ptr, ptr, idx, cnt, 16,
        ws_bytes, None)
    assert ftk(vl, tok, None, 16) == L.HS_ERR_INVALID_ARG
    assert ftk(vl, tok, 16, None) == L.HS_ERR_INVALID_ARG
    assert ftk(None, tok, 16, 16) == L.HS_ERR_INVALID_ARG
    assert ftk(vl, tok, 16, 16, ptr=None) == L.HS_ERR_INVALID_ARG
    assert ftk(vl, tok, 16, 16, ptr=18) == L.HS_ERR_INVALID_ARG          # misaligned
    assert ftk(vl, tok, 16, 16, ws_bytes=8) == L.HS_ERR_WORKSPACE
    assert ftk(vl, L.HsSel(16, 1, 5000, 32), 16, 16) == L.HS_ERR_UNSUPPORTED
    # unknown selection flags are rejected
    bad = L.HsSel(16, 16, 8, 32, 2)
    assert _call_full(lib, vl, bad) == L.HS_ERR_INVALID_ARG
    # exp2 self test: empty is a no-op, null / misaligned / negative sizes are rejected before launch
    assert lib.hs_debug_exp2_poly(None, None, 0, None) == L.HS_OK
    assert lib.hs_debug_exp2_poly(None, None, 4, None) == L.HS_ERR_INVALID_ARG
    assert lib.hs_debug_exp2_poly(16, 18, 4, None) == L.HS_ERR_INVALID_ARG
    assert lib.hs_debug_exp2_poly(16, 32, -1, None) == L.HS_ERR_INVALID_ARG


def test_batch_without_new_tokens_returns_before_touching_pointers(lib):
    """Sequences with no new tokens: every call returns HS_OK on the host with
    null data, index and workspace pointers (nothing is launched)."""
    from hybrid_sparse_attention_tma_b200 import _lib as L
    vl = _varlen([0, 0, 0], [0, 64, 164], hq=64, hkv=1, d=128)
    dec = L.HsSel(1, 1, 16, 8)
    blk = L.HsSel(64, 64, 2, 0)
    n = None
    assert lib.hs_full_attn_select(ctypes.byref(vl), ctypes.byref(blk), n, n, n, n, n, n, n, 0, n) == L.HS_OK
    assert lib.hs_topk_select(ctypes.byref(vl), ctypes.byref(blk), n, n, n, n, 0, n) == L.HS_OK
    for s_ in (blk, L.HsSel(64, 1, 1024, 128)):
        assert lib.hs_full_attn_select_topk(ctypes.byref(vl), ctypes.byref(s_), n, n, n, n, n, n, n, n, n, 0,
                                            n) == L.HS_OK
    assert lib.hs_sparse_attn_prefill(ctypes.byref(vl), ctypes.byref(blk), n, n, n, n, n, n, n, n, 0, n) == L.HS_OK
    assert lib.hs_sparse_swa_gated_prefill(ctypes.byref(vl), ctypes.byref(blk), n, n, n, n, n, 128, n, n, n, n, n,
                                           n, n, 0, n) == L.HS_OK
    assert lib.hs_swa_gated(ctypes.byref(vl), 128, n, n, n, n, n, n, n, 0, n) == L.HS_OK
    assert lib.hs_sparse_attn_decode(ctypes.byref(vl), ctypes.byref(dec), n, L.HS_KV_BF16, n, n, n, n, n, n, 0, n, n,
                                     n, 0, n) == L.HS_OK
    # a batch of no sequences at all is malformed
    assert lib.hs_sparse_attn_decode(ctypes.byref(_varlen([0], [0], hq=64, hkv=1, d=128)), ctypes.byref(dec), n,
                                     L.HS_KV_BF16, n, n, n, n, n, n, 0, n, n, n, 0, n) == L.HS_ERR_INVALID_ARG


def test_workspace_size_every_op_at_workload_shapes(lib):
    """Every op sizes a workspace (header + scratch) for the benchmarked shapes."""
    import workloads as W
    from hybrid_sparse_attention_tma_b200 import _lib as L
    ops = [L.HS_OP_FULL_ATTN_SELECT, L.HS_OP_TOPK_SELECT, L.HS_OP_SPARSE_ATTN_PREFILL, L.HS_OP_SPARSE_ATTN_DECODE,
           L.HS_OP_SWA_GATED, L.HS_OP_SPARSE_SWA_GATED_PREFILL]
    for name in ["tiny", "hys_block", "hys2_prefill", "decode", "agentic"]:
        w = W.WORKLOADS[name]
        vl = _varlen(w.cu_q(), w.cu_kv(), hq=w.n_q_heads, hkv=w.n_kv_heads, d=w.head_dim)
        sel = L.HsSel(w.q_tile, w.block, w.topk, w.window)
        for op in ops:
            if op == L.HS_OP_SPARSE_ATTN_DECODE and name != "decode":
                continue
            n = lib.hs_workspace_size(op, ctypes.byref(vl), ctypes.byref(sel))
            assert n >= 256 and n % 256 == 0, (name, op, n)
        if name == "hys_block":  # the block-max spill: one double-buffered share per SM, whole 128-key tiles
            n = lib.hs_workspace_size(L.HS_OP_FULL_ATTN_SELECT, ctypes.byref(vl), ctypes.byref(sel))
            assert n >= 2 * (w.max_kv // 128) * (128 // w.block) * 256 * 4


def test_bench_traffic_needs_matching_source_hash(tmp_path, monkeypatch):
    import json
    import sys
    sys.path.insert(0, ROOT)
    import bench
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    for f in bench.KERNEL_SOURCES:  # the hash is taken over the kernel sources under ROOT
        dst = tmp_path / f
        dst.parent.mkdir(parents=True, exist_ok=True)
        with open(os.path.join(ROOT, f), "rb") as fh:
            dst.write_bytes(fh.read())
    h = bench.src_hash()
    (prof / "traffic.json").write_text(json.dumps({"attn_fwd_full:hys_block": {"src_hash": h,
                                                                                "dram_bytes_per_launch": 123}}))
    assert bench.traffic_for("attn_fwd_full", "hys_block") == 123
    assert bench.traffic_for("attn_fwd_full", "decode") is None
    (prof / "traffic.json").write_text(json.dumps({"attn_fwd_full:hys_block": {"src_hash": "stale",
                                                                                "dram_bytes_per_launch": 123}}))
    assert bench.traffic_for("attn_fwd_full", "hys_block") is None


def test_cpu_baseline_samples_until_the_time_budget():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    w = W.WORKLOADS["tiny"]
    toks, times = bench.time_oracle(w, min_seconds=1e-6, max_tiles=3)
    assert len(toks) == 1 and toks[0] == w.q_tile  # one middle tile already exceeds a tiny budget
    toks, times = bench.time_oracle(w, min_seconds=1e9, max_tiles=3)
    assert len(toks) == 3 and all(t > 0 for t in times)  # capped by max_tiles
    toks, times = bench.time_oracle(w, 2, repeats=2)
    assert toks == 2 * w.q_tile and len(times) == 2


def test_clock_summary_median_max_and_reasons():
    sys.path.insert(0, ROOT)
    import bench
    lines = ["0, 1965, 1965, 610.2, 0x0, Not Active, Not Active, Not Active, Not Active\n",
             "0, 1755, 1965, 998.7, 0x4, Not Active, Not Active, Not Active, Active\n",
             "0, 1740, 1965, 1001.0, 0x4, Not Active, Not Active, Not Active, Active\n",
             "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active\n",
             "garbage\n"]
    c = bench.summarize_clocks(lines)
    assert c == {"sm_mhz": 1755.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    c = bench.summarize_clocks(["0, 1200, 1965, 700, 0x8, Active, Not Active, Active, Not Active\n"])
    assert c["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]
    assert bench.summarize_clocks([]) is None


def test_reference_arm_prints_the_contract_line():
    """bench.py --impl reference: the oracle on the host cores, one JSON line
    with the keys the driver reads (tiny workload, so it runs in seconds)."""
    import json
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                          "tiny", "--steps", "2", "--warmup", "3"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ["impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"]:
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
