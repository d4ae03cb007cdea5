"""libhs: hybrid-block sparse attention (HySparse / HySparse2) on B200.

Thin Python binding over the C ABI in include/hs.h. Every step of the path runs
in libhs's CUDA kernels; this module only allocates outputs/workspaces with
torch, builds the argument structs and checks status codes. There is no
fallback: if libhs.so is missing the import of the library raises.
"""
from __future__ import annotations

import ctypes
import math
from typing import List, Optional, Sequence

import torch

from . import _lib as L
from ._lib import HsError, HS_KV_BF16, HS_KV_FP8_E4M3  # noqa: F401

__all__ = ["Varlen", "Sel", "Workspace", "full_attn_select", "full_attn_select_topk", "topk_select", "sparse_attn_prefill",
           "gather_selected_kv", "sparse_attn_decode", "swa_gated", "sparse_swa_gated_prefill", "kv_dequantize",
           "swa_ring_write", "swa_gated_decode",
           "workspace_size", "check_error", "HsError"]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Varlen:
    """Packed variable-length batch: prefix sums of new queries and of keys."""

    def __init__(self, cu_q: Sequence[int], cu_kv: Sequence[int], n_q_heads: int, n_kv_heads: int,
                 head_dim: int, device="cuda", softmax_scale: float = 0.0):
        self.cu_q_list: List[int] = [int(x) for x in cu_q]
        self.cu_kv_list: List[int] = [int(x) for x in cu_kv]
        self.batch = len(self.cu_q_list) - 1
        self.n_q_heads, self.n_kv_heads, self.head_dim = n_q_heads, n_kv_heads, head_dim
        self.cu_q = torch.tensor(self.cu_q_list, dtype=torch.int32, device=device)
        self.cu_kv = torch.tensor(self.cu_kv_list, dtype=torch.int32, device=device)
        self._hq = (ctypes.c_int32 * len(self.cu_q_list))(*self.cu_q_list)
        self._hkv = (ctypes.c_int32 * len(self.cu_kv_list))(*self.cu_kv_list)
        self.c = L.HsVarlen(self.batch, n_q_heads, n_kv_heads, head_dim,
                            self.cu_q.data_ptr(), self.cu_kv.data_ptr(), self._hq, self._hkv,
                            float(softmax_scale))

    @property
    def total_q(self) -> int:
        return self.cu_q_list[-1]

    @property
    def total_kv(self) -> int:
        return self.cu_kv_list[-1]

    @property
    def max_kv(self) -> int:
        return max(b - a for a, b in zip(self.cu_kv_list, self.cu_kv_list[1:]))

    def n_tiles(self, T: int) -> int:
        return sum((b - a + T - 1) // T for a, b in zip(self.cu_q_list, self.cu_q_list[1:]))


def Sel(q_tile: int, block: int, topk: int, window: int, exclusive: bool = False) -> L.HsSel:
    """Selection parameters; exclusive=True draws the top-k only from blocks
    that end before the forced window of the tile's last query."""
    return L.HsSel(q_tile, block, topk, window, L.HS_SEL_WINDOW_EXCLUSIVE if exclusive else 0)


def workspace_size(op: int, vl: Varlen, sel: Optional[L.HsSel] = None) -> int:
    lib = L.load()
    n = lib.hs_workspace_size(op, ctypes.byref(vl.c), ctypes.byref(sel) if sel is not None else None)
    if n == 0:
        raise HsError("hs_workspace_size", L.HS_ERR_INVALID_ARG, "invalid shapes")
    return n


class Workspace:
    """Caller-owned device scratch; grows on demand; header zeroed once."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf: Optional[torch.Tensor] = None

    def get(self, nbytes: int, stream=None) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
            L.check("hs_workspace_init", L.load().hs_workspace_init(_ptr(self.buf), self.buf.numel(), _stream(stream)))
        return self.buf


_default_ws = {}


def _ws(ws: Optional[Workspace], device) -> Workspace:
    if ws is not None:
        return ws
    key = str(device)
    if key not in _default_ws:
        _default_ws[key] = Workspace(device)
    return _default_ws[key]


def check_error(ws: Workspace, stream=None):
    """Synchronise and raise if a device-side bounded wait gave up."""
    L.check("hs_check_error", L.load().hs_check_error(_ptr(ws.buf), _stream(stream)))


def full_attn_select(vl: Varlen, sel: L.HsSel, q, k, v, o=None, lse=None, scores=None,
                     ws: Optional[Workspace] = None, stream=None):
    """Full causal attention + importance scores. Returns (o, lse, scores)."""
    lib = L.load()
    dev = q.device
    Tq, Hq, d = q.shape
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((Hq, Tq), dtype=torch.float32, device=dev) if lse is None else lse
    nblk = (vl.max_kv + sel.block - 1) // sel.block
    if scores is None:
        scores = torch.empty((vl.n_tiles(sel.q_tile), vl.n_kv_heads, nblk), dtype=torch.float32, device=dev)
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_FULL_ATTN_SELECT, vl, sel), stream)
    L.check("hs_full_attn_select", lib.hs_full_attn_select(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(scores),
        _ptr(buf), buf.numel(), _stream(stream)))
    return o, lse, scores


def full_attn_select_topk(vl: Varlen, sel: L.HsSel, q, k, v, o=None, lse=None, scores=None, idx=None, cnt=None,
                          ws: Optional[Workspace] = None, stream=None):
    """Full layer and top-k in one call: (o, lse, idx, cnt) equal to those of
    full_attn_select followed by topk_select. Token-level prefill takes the
    top-k inside the score pass (`scores` is then scratch with undefined
    content); other shapes run the two calls. Returns (o, lse, idx, cnt)."""
    lib = L.load()
    dev = q.device
    Tq, Hq, d = q.shape
    o = torch.empty_like(q) if o is None else o
    lse = torch.empty((Hq, Tq), dtype=torch.float32, device=dev) if lse is None else lse
    nblk = (vl.max_kv + sel.block - 1) // sel.block
    nt = vl.n_tiles(sel.q_tile)
    if scores is None:
        scores = torch.empty((nt, vl.n_kv_heads, nblk), dtype=torch.float32, device=dev)
    idx = torch.empty((nt, vl.n_kv_heads, max(sel.topk, 1)), dtype=torch.int32, device=dev) if idx is None else idx
    cnt = torch.empty((nt, vl.n_kv_heads), dtype=torch.int32, device=dev) if cnt is None else cnt
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_FULL_ATTN_SELECT, vl, sel), stream)
    L.check("hs_full_attn_select_topk", lib.hs_full_attn_select_topk(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(scores),
        _ptr(idx), _ptr(cnt), _ptr(buf), buf.numel(), _stream(stream)))
    return o, lse, idx, cnt


def topk_select(vl: Varlen, sel: L.HsSel, scores, idx=None, cnt=None, ws: Optional[Workspace] = None,
                stream=None):
    """Top-k candidate blocks per (tile, KV head). Returns (idx, cnt)."""
    lib = L.load()
    dev = scores.device
    nt = vl.n_tiles(sel.q_tile)
    idx = torch.empty((nt, vl.n_kv_heads, max(sel.topk, 1)), dtype=torch.int32, device=dev) if idx is None else idx
    cnt = torch.empty((nt, vl.n_kv_heads), dtype=torch.int32, device=dev) if cnt is None else cnt
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_TOPK_SELECT, vl, sel), stream)
    L.check("hs_topk_select", lib.hs_topk_select(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(scores), _ptr(idx), _ptr(cnt), _ptr(buf), buf.numel(),
        _stream(stream)))
    return idx, cnt


def sparse_attn_prefill(vl: Varlen, sel: L.HsSel, q, k, v, idx, cnt, o=None, lse=None,
                        ws: Optional[Workspace] = None, stream=None, want_lse: bool = True, kg=None, vg=None):
    """Sparse layer over the reused KV cache and indices. Returns (o, lse).
    With kg / vg from gather_selected_kv (token-level selection) the selected
    rows are read from those buffers (same result)."""
    lib = L.load()
    dev = q.device
    Tq, Hq, d = q.shape
    o = torch.empty_like(q) if o is None else o
    if lse is None and want_lse:
        lse = torch.empty((Hq, Tq), dtype=torch.float32, device=dev)
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_SPARSE_ATTN_PREFILL, vl, sel), stream)
    if kg is not None:
        L.check("hs_sparse_attn_prefill_gathered", lib.hs_sparse_attn_prefill_gathered(
            ctypes.byref(vl.c), ctypes.byref(sel), _ptr(q), _ptr(k), _ptr(v), _ptr(kg), _ptr(vg), _ptr(idx),
            _ptr(cnt), _ptr(o), _ptr(lse), _ptr(buf), buf.numel(), _stream(stream)))
        return o, lse
    L.check("hs_sparse_attn_prefill", lib.hs_sparse_attn_prefill(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt), _ptr(o),
        _ptr(lse), _ptr(buf), buf.numel(), _stream(stream)))
    return o, lse


def gather_selected_kv(vl: Varlen, sel: L.HsSel, k, v, idx, cnt, kg=None, vg=None, stream=None):
    """Token-level selection: the selected tokens' K / V rows of every
    (selection tile, KV head), [n_tiles, H_kv, topk, d], zero past cnt; once
    per block, read by every sparse prefill layer. Returns (kg, vg)."""
    lib = L.load()
    shape = (vl.n_tiles(sel.q_tile), vl.n_kv_heads, max(sel.topk, 1), k.shape[-1])
    kg = torch.empty(shape, dtype=k.dtype, device=k.device) if kg is None else kg
    vg = torch.empty(shape, dtype=v.dtype, device=v.device) if vg is None else vg
    L.check("hs_gather_selected_kv", lib.hs_gather_selected_kv(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt), _ptr(kg), _ptr(vg),
        _stream(stream)))
    return kg, vg


def sparse_swa_gated_prefill(vl: Varlen, sel: L.HsSel, q, k, v, idx, cnt, swa_window: int, k_swa, v_swa, gamma,
                             o=None, o_sparse=None, lse_sparse=None, ws: Optional[Workspace] = None, stream=None):
    """A whole HySparse sparse layer in one launch: block-sparse branch over the
    reused cache, own-cache sliding window, sigmoid gate. o_sparse / lse_sparse
    are written only when given. Returns o."""
    lib = L.load()
    dev = q.device
    o = torch.empty_like(q) if o is None else o
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_SPARSE_SWA_GATED_PREFILL, vl, sel), stream)
    L.check("hs_sparse_swa_gated_prefill", lib.hs_sparse_swa_gated_prefill(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt), swa_window,
        _ptr(k_swa), _ptr(v_swa), _ptr(gamma), _ptr(o), _ptr(o_sparse), _ptr(lse_sparse), _ptr(buf), buf.numel(),
        _stream(stream)))
    return o


def sparse_attn_decode(vl: Varlen, sel: L.HsSel, q, k, v, idx, cnt, k_scale=None, v_scale=None,
                       kv_dtype: int = HS_KV_BF16, split_k: int = 0, o=None, lse=None,
                       ws: Optional[Workspace] = None, stream=None):
    """Sparse decode (one query per sequence), bf16 or FP8-e4m3 KV. Returns (o, lse)."""
    lib = L.load()
    dev = q.device
    Tq, Hq, d = q.shape
    o = torch.empty((Tq, Hq, d), dtype=torch.bfloat16, device=dev) if o is None else o
    lse = torch.empty((Hq, Tq), dtype=torch.float32, device=dev) if lse is None else lse
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_SPARSE_ATTN_DECODE, vl, sel), stream)
    L.check("hs_sparse_attn_decode", lib.hs_sparse_attn_decode(
        ctypes.byref(vl.c), ctypes.byref(sel), _ptr(q), kv_dtype, _ptr(k), _ptr(v), _ptr(k_scale),
        _ptr(v_scale), _ptr(idx), _ptr(cnt), split_k, _ptr(o), _ptr(lse), _ptr(buf), buf.numel(),
        _stream(stream)))
    return o, lse


def kv_dequantize(codes, scale, out=None, stream=None):
    """FP8-e4m3 KV codes [T, H, d] uint8 with scales [T, H] fp32 -> bf16 [T, H, d]."""
    lib = L.load()
    T, H, d = codes.shape
    out = torch.empty((T, H, d), dtype=torch.bfloat16, device=codes.device) if out is None else out
    L.check("hs_kv_dequantize", lib.hs_kv_dequantize(_ptr(codes), _ptr(scale), T * H, d, _ptr(out), _stream(stream)))
    return out


def swa_ring_write(vl: Varlen, k_new, v_new, k_ring, v_ring, stream=None):
    """Store the new tokens' rows [T_q, H_kv, d] of a layer's own SWA cache in
    its rings [batch, R, H_kv, d] (position p at slot p mod R)."""
    lib = L.load()
    L.check("hs_swa_ring_write", lib.hs_swa_ring_write(
        ctypes.byref(vl.c), k_ring.shape[1], _ptr(k_new), _ptr(v_new), _ptr(k_ring), _ptr(v_ring), _stream(stream)))
    return k_ring, v_ring


def swa_gated_decode(vl: Varlen, window: int, q, k_ring, v_ring, gamma, o_sparse, o=None, stream=None):
    """Decode: the own-cache sliding-window branch over the rings and the
    sigmoid gate with the sparse branch. Returns o."""
    lib = L.load()
    o = torch.empty_like(q) if o is None else o
    L.check("hs_swa_gated_decode", lib.hs_swa_gated_decode(
        ctypes.byref(vl.c), window, k_ring.shape[1], _ptr(q), _ptr(k_ring), _ptr(v_ring), _ptr(gamma),
        _ptr(o_sparse), _ptr(o), _stream(stream)))
    return o


def swa_gated(vl: Varlen, window: int, q, k_swa, v_swa, gamma, o_sparse, o=None,
              ws: Optional[Workspace] = None, stream=None):
    """Own-cache sliding-window branch fused with the sigmoid gate. Returns o."""
    lib = L.load()
    dev = q.device
    o = torch.empty_like(q) if o is None else o
    w = _ws(ws, dev)
    buf = w.get(workspace_size(L.HS_OP_SWA_GATED, vl, None), stream)
    L.check("hs_swa_gated", lib.hs_swa_gated(
        ctypes.byref(vl.c), window, _ptr(q), _ptr(k_swa), _ptr(v_swa), _ptr(gamma), _ptr(o_sparse), _ptr(o),
        _ptr(buf), buf.numel(), _stream(stream)))
    return o
