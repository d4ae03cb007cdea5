"""ctypes view of include/hs.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhs.so")

HS_OK, HS_ERR_INVALID_ARG, HS_ERR_UNSUPPORTED, HS_ERR_WORKSPACE, HS_ERR_CUDA, HS_ERR_TIMEOUT = range(6)
(HS_OP_FULL_ATTN_SELECT, HS_OP_TOPK_SELECT, HS_OP_SPARSE_ATTN_PREFILL, HS_OP_SPARSE_ATTN_DECODE, HS_OP_SWA_GATED,
 HS_OP_SPARSE_SWA_GATED_PREFILL) = range(6)
HS_KV_BF16, HS_KV_FP8_E4M3 = 0, 1

# Every function the header declares; the CPU test checks the library exports them all.
EXPORTS = [
    "hs_workspace_size", "hs_workspace_init", "hs_check_error", "hs_status_string",
    "hs_full_attn_select", "hs_full_attn_select_topk", "hs_topk_select", "hs_sparse_attn_prefill",
    "hs_sparse_attn_decode", "hs_swa_gated", "hs_debug_wait_timeout", "hs_last_error_detail",
    "hs_full_attn_select_noalloc", "hs_sparse_swa_gated_prefill", "hs_debug_exp2_poly", "hs_kv_dequantize",
    "hs_gather_selected_kv", "hs_sparse_attn_prefill_gathered", "hs_swa_ring_write", "hs_swa_gated_decode",
]


class HsVarlen(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("cu_q", ctypes.c_void_p), ("cu_kv", ctypes.c_void_p),
        ("cu_q_host", ctypes.POINTER(ctypes.c_int32)), ("cu_kv_host", ctypes.POINTER(ctypes.c_int32)),
        ("softmax_scale", ctypes.c_float),
    ]


class HsSel(ctypes.Structure):
    _fields_ = [("q_tile", ctypes.c_int32), ("block", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("window", ctypes.c_int32), ("flags", ctypes.c_int32)]


HS_SEL_WINDOW_EXCLUSIVE = 1


class HsError(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


_lib = None


def load():
    """Load libhs.so; raise loudly if it is not built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libhs.so is not built at {LIB_PATH}; run `python -m hybrid_sparse_attention_tma_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
    VL, SEL = ctypes.POINTER(HsVarlen), ctypes.POINTER(HsSel)
    lib.hs_workspace_size.restype = sz
    lib.hs_workspace_size.argtypes = [ctypes.c_int, VL, SEL]
    lib.hs_workspace_init.restype = i32
    lib.hs_workspace_init.argtypes = [vp, sz, vp]
    lib.hs_check_error.restype = i32
    lib.hs_check_error.argtypes = [vp, vp]
    lib.hs_status_string.restype = ctypes.c_char_p
    lib.hs_status_string.argtypes = [i32]
    lib.hs_full_attn_select.restype = i32
    lib.hs_full_attn_select.argtypes = [VL, SEL, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hs_full_attn_select_topk.restype = i32
    lib.hs_full_attn_select_topk.argtypes = [VL, SEL, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hs_topk_select.restype = i32
    lib.hs_topk_select.argtypes = [VL, SEL, vp, vp, vp, vp, sz, vp]
    lib.hs_sparse_attn_prefill.restype = i32
    lib.hs_sparse_attn_prefill.argtypes = [VL, SEL, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hs_gather_selected_kv.restype = i32
    lib.hs_gather_selected_kv.argtypes = [VL, SEL, vp, vp, vp, vp, vp, vp, vp]
    lib.hs_swa_ring_write.restype = i32
    lib.hs_swa_ring_write.argtypes = [VL, i32, vp, vp, vp, vp, vp]
    lib.hs_swa_gated_decode.restype = i32
    lib.hs_swa_gated_decode.argtypes = [VL, i32, i32, vp, vp, vp, vp, vp, vp, vp]
    lib.hs_sparse_attn_prefill_gathered.restype = i32
    lib.hs_sparse_attn_prefill_gathered.argtypes = [VL, SEL, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hs_sparse_attn_decode.restype = i32
    lib.hs_sparse_attn_decode.argtypes = [VL, SEL, vp, i32, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp, sz, vp]
    lib.hs_swa_gated.restype = i32
    lib.hs_swa_gated.argtypes = [VL, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hs_sparse_swa_gated_prefill.restype = i32
    lib.hs_sparse_swa_gated_prefill.argtypes = [VL, SEL, vp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.hs_full_attn_select_noalloc.restype = i32
    lib.hs_full_attn_select_noalloc.argtypes = [VL, SEL, vp, vp, vp, vp, vp, vp, i32, vp]
    lib.hs_last_error_detail.restype = i32
    lib.hs_last_error_detail.argtypes = [ctypes.POINTER(i32)] * 3
    lib.hs_debug_wait_timeout.restype = i32
    lib.hs_debug_wait_timeout.argtypes = [vp, sz, ctypes.c_uint64, vp]
    lib.hs_debug_exp2_poly.restype = i32
    lib.hs_debug_exp2_poly.argtypes = [vp, vp, ctypes.c_int64, vp]
    lib.hs_kv_dequantize.restype = i32
    lib.hs_kv_dequantize.argtypes = [vp, vp, ctypes.c_int64, i32, vp, vp]
    _lib = lib
    return lib


def check(fn: str, status: int):
    if status != HS_OK:
        lib = load()
        msg = lib.hs_status_string(status).decode()
        if status == HS_ERR_TIMEOUT:
            a, b, c = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
            lib.hs_last_error_detail(ctypes.byref(a), ctypes.byref(b), ctypes.byref(c))
            msg += f"; site {a.value}, block {b.value}, item {c.value >> 12}, step {c.value & 0xFFF}"
        raise HsError(fn, status, msg)
