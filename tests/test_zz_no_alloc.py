"""The allocation-free full-attention entry point against the workspace one.

hs_full_attn_select_noalloc serves callers that cannot allocate device memory
(a plugin inside a runtime that owns all device memory, or a path that must
not call cudaMalloc): it uses a fixed array inside the library instead of a
caller workspace. This test calls it through the C ABI twice in a row (the
second call reuses the array's leftover contents) and checks O, lse and the
block scores against hs_full_attn_select with the tolerances of the other
parity tests. It lives in its own file so it runs last in a full session and
also passes alone in a fresh process.
"""
import ctypes

import pytest
import torch

import workloads as W
from tests.parity import f64, assert_close_out, assert_close_lse, assert_scores_close

pytestmark = pytest.mark.gpu


def _noalloc(lib, vl, sel, q, k, v, o, lse, scores):
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return lib.hs_full_attn_select_noalloc(ctypes.byref(vl.c), ctypes.byref(sel), P(q), P(k), P(v), P(o), P(lse),
                                           P(scores), 1, s)


def test_noalloc_matches_workspace_entry_point_twice():
    from hybrid_sparse_attention_tma_b200 import build
    build.build()
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200 import _lib as L
    lib = L.load()
    # ragged chunked prefill, GQA group 4, d = 128, 64-token blocks: several
    # work items per CTA and both Q tiles of an item in use
    w = W.Workload("noalloc", ctx=(0, 700), new=(1500, 900), n_q_heads=16, n_kv_heads=4, head_dim=128,
                   q_tile=64, block=64, topk=8, window=0, n_sparse=0)
    inp = W.make_block_inputs(w, device="cuda", seed=21)
    vl = hs.Varlen(w.cu_q(), w.cu_kv(), w.n_q_heads, w.n_kv_heads, w.head_dim, device="cuda")
    sel = hs.Sel(w.q_tile, w.block, w.topk, w.window)
    o_ref, lse_ref, sc_ref = hs.full_attn_select(vl, sel, inp.q, inp.k, inp.v)
    torch.cuda.synchronize()
    for _ in range(2):
        o = torch.full_like(o_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        sc = torch.full_like(sc_ref, -1.0)
        assert _noalloc(lib, vl, sel, inp.q, inp.k, inp.v, o, lse, sc) == L.HS_OK
        torch.cuda.synchronize()
        assert_close_out(f64(o), f64(o_ref), what="noalloc o")
        assert_close_lse(f64(lse), f64(lse_ref), what="noalloc lse")
        assert_scores_close(f64(sc), f64(sc_ref), range(sc_ref.shape[0]), what="noalloc scores")


def test_noalloc_rejects_oversized_problem_before_launch():
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200 import _lib as L
    lib = L.load()
    # 32768 blocks of 8 keys would need 64 MiB for a single CTA's double-buffered spill
    n = 8 * 32768
    vl = hs.Varlen([0, 1], [0, n], 4, 1, 64, device="cuda")
    sel = hs.Sel(16, 8, 8, 0)
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    P = ctypes.c_void_p(dummy.data_ptr())
    st = lib.hs_full_attn_select_noalloc(ctypes.byref(vl.c), ctypes.byref(sel), P, P, P, P, P, P, 1, None)
    assert st == L.HS_ERR_WORKSPACE
