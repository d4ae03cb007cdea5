"""One hybrid block: a full attention layer feeding N sparse layers that reuse
its KV cache and its top-k indices (QbitAI repost of HySparse, "hybrid block";
HySparse2 release note, "KV Reuse"). HySparse sparse layers also run the
own-cache sliding-window branch and the sigmoid gate.

Only sequencing of library calls lives here; all arithmetic is in libhs.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import torch

from . import (Varlen, Sel, Workspace, full_attn_select, full_attn_select_topk, topk_select, sparse_attn_prefill,
               sparse_attn_decode,
               swa_gated, sparse_swa_gated_prefill, kv_dequantize, gather_selected_kv, swa_gated_decode,
               swa_ring_write, HS_KV_BF16, HS_KV_FP8_E4M3)


@dataclass
class SparseLayerIn:
    q: torch.Tensor                       # [T_q, H_q, d] bf16, this layer's queries
    k_swa: Optional[torch.Tensor] = None  # own SWA cache (HySparse): prefill [T_kv, H_kv, d] bf16;
    #   decode: the ring [batch, R, H_kv, d] (hs_swa_ring_write), R >= the window
    v_swa: Optional[torch.Tensor] = None
    gamma: Optional[torch.Tensor] = None  # [T_q, H_q] fp32 gate logits


class HybridBlock:
    def __init__(self, vl: Varlen, q_tile: int, block: int, topk: int, window: int, swa_window: int = 0,
                 device="cuda", fused: bool = True, exclusive: bool = False, fuse_topk: bool = False):
        self.vl = vl
        self.sel = Sel(q_tile, block, topk, window, exclusive)
        self.swa_window = swa_window
        # prefill layers with a window branch run as one fused launch
        # (hs_sparse_swa_gated_prefill) unless fused=False (two launches)
        self.fused = fused
        self.ws = Workspace(device)
        self.device = device
        self._bufs = {}
        # one query per sequence with single-query tiles: the sparse layers use
        # the decode path (token- or block-level selection; a window branch
        # reads the layer's own cache as a ring)
        self.decode = q_tile == 1 and all(b - a == 1 for a, b in zip(vl.cu_q_list, vl.cu_q_list[1:]))
        # token-level prefill: the selected rows are gathered once per block
        # (hs_gather_selected_kv) and every plain sparse layer reads them
        self.gathered = (not self.decode and block == 1 and topk > 0 and not (swa_window > 0 and fused))
        # token-level prefill with fuse_topk=True: the top-k is taken inside the
        # score pass (hs_full_attn_select_topk; the scores then stay scratch).
        # The default runs the full layer, then hs_topk_select on the stored
        # scores, which measures faster on B200 (the selection competes with
        # the score pass for its SMs more than the separate launch costs).
        self.fuse_topk = fuse_topk and block == 1 and not self.decode

    def swa_rings(self, k_swa, v_swa, stream=None):
        """Decode: a layer's own window cache [T_kv, H_kv, d] (all positions, in
        cu_kv order) as the rings [batch, swa_window, H_kv, d] the decode path
        reads (hs_swa_ring_write with every cached token new: the last
        swa_window positions of each sequence land at slot p mod swa_window)."""
        vl = self.vl
        every = Varlen(vl.cu_kv_list, vl.cu_kv_list, vl.n_q_heads, vl.n_kv_heads, vl.head_dim, device=self.device)
        shape = (vl.batch, self.swa_window, vl.n_kv_heads, vl.head_dim)
        kr = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        vr = torch.zeros(shape, dtype=torch.bfloat16, device=self.device)
        swa_ring_write(every, k_swa, v_swa, kr, vr, stream=stream)
        return kr, vr

    def _buf(self, name, shape, dtype):
        t = self._bufs.get(name)
        if t is None or t.shape != torch.Size(shape) or t.dtype != dtype:
            t = torch.empty(shape, dtype=dtype, device=self.device)
            self._bufs[name] = t
        return t

    def forward(self, q, k, v, layers: List[SparseLayerIn], stream=None, keep_all: bool = False, fp8_kv=None,
                intermediates: bool = True, layer_hook=None):
        """Returns dict(o_full, lse_full, scores, idx, cnt, layers=[{o_sparse, lse_sparse, o}]).
        scores is None when the top-k ran inside the score pass (fuse_topk).

        With keep_all=False, output buffers are reused across calls (no
        allocation in steady state) and only the last layer's tensors are
        guaranteed distinct. fp8_kv = (k_codes, v_codes, k_scale, v_scale) makes the
        sparse decode layers read an FP8-e4m3 copy of the KV cache; in prefill
        the block reads that FP8 cache everywhere: it is expanded to bf16 once
        (hs_kv_dequantize) and the full and sparse layers use the expansion
        (k and v may then be None). With
        intermediates=False a fused layer does not write o_sparse / lse_sparse
        (they are returned as None). layer_hook (see forward_from_host) supplies
        each layer's inputs just before its launches and is told when they are
        enqueued."""
        vl, sel = self.vl, self.sel
        Tq, Hq, d = q.shape
        nblk = (vl.max_kv + sel.block - 1) // sel.block
        nt = vl.n_tiles(sel.q_tile)
        o = self._buf("o_full", (Tq, Hq, d), torch.bfloat16)
        lse = self._buf("lse_full", (Hq, Tq), torch.float32)
        scores = self._buf("scores", (nt, vl.n_kv_heads, nblk), torch.float32)
        idx = self._buf("idx", (nt, vl.n_kv_heads, max(sel.topk, 1)), torch.int32)
        cnt = self._buf("cnt", (nt, vl.n_kv_heads), torch.int32)
        if fp8_kv is not None and not self.decode:
            kq, vq, ks, vs = fp8_kv
            k = kv_dequantize(kq, ks, self._buf("k_deq", tuple(kq.shape), torch.bfloat16), stream=stream)
            v = kv_dequantize(vq, vs, self._buf("v_deq", tuple(vq.shape), torch.bfloat16), stream=stream)
        if self.fuse_topk:
            full_attn_select_topk(vl, sel, q, k, v, o, lse, scores, idx, cnt, ws=self.ws, stream=stream)
        else:
            full_attn_select(vl, sel, q, k, v, o, lse, scores, ws=self.ws, stream=stream)
            topk_select(vl, sel, scores, idx, cnt, ws=self.ws, stream=stream)
        kg = vg = None
        if self.gathered and layers:
            gshape = (nt, vl.n_kv_heads, sel.topk, d)
            kg, vg = gather_selected_kv(vl, sel, k, v, idx, cnt, self._buf("kg", gshape, torch.bfloat16),
                                        self._buf("vg", gshape, torch.bfloat16), stream=stream)
        outs = []
        for i, L in enumerate(layers):
            if layer_hook is not None:
                L = layer_hook.before(i)  # this layer's inputs, once they are on the device
            tag = str(i) if keep_all else str(i % 2)
            o_sp = self._buf("o_sp" + tag, (Tq, Hq, d), torch.bfloat16)
            lse_sp = self._buf("lse_sp" + tag, (Hq, Tq), torch.float32)
            if self.decode:
                if fp8_kv is not None:
                    kq, vq, ks, vs = fp8_kv
                    sparse_attn_decode(vl, sel, L.q, kq, vq, idx, cnt, ks, vs, HS_KV_FP8_E4M3, o=o_sp, lse=lse_sp,
                                       ws=self.ws, stream=stream)
                else:
                    sparse_attn_decode(vl, sel, L.q, k, v, idx, cnt, kv_dtype=HS_KV_BF16, o=o_sp, lse=lse_sp,
                                       ws=self.ws, stream=stream)
            elif not (self.swa_window > 0 and self.fused):
                sparse_attn_prefill(vl, sel, L.q, k, v, idx, cnt, o_sp, lse_sp, ws=self.ws, stream=stream,
                                    kg=kg, vg=vg)
            if self.swa_window > 0 and self.fused and not self.decode:
                o_l = self._buf("o_l" + tag, (Tq, Hq, d), torch.bfloat16)
                if not intermediates:
                    o_sp = lse_sp = None
                sparse_swa_gated_prefill(vl, sel, L.q, k, v, idx, cnt, self.swa_window, L.k_swa, L.v_swa, L.gamma,
                                         o=o_l, o_sparse=o_sp, lse_sparse=lse_sp, ws=self.ws, stream=stream)
            elif self.swa_window > 0 and self.decode:
                o_l = self._buf("o_l" + tag, (Tq, Hq, d), torch.bfloat16)
                swa_gated_decode(vl, self.swa_window, L.q, L.k_swa, L.v_swa, L.gamma, o_sp, o_l, stream=stream)
            elif self.swa_window > 0:
                o_l = self._buf("o_l" + tag, (Tq, Hq, d), torch.bfloat16)
                swa_gated(vl, self.swa_window, L.q, L.k_swa, L.v_swa, L.gamma, o_sp, o_l, ws=self.ws,
                          stream=stream)
            else:
                o_l = o_sp
            outs.append({"o_sparse": o_sp, "lse_sparse": lse_sp, "o": o_l})
            if layer_hook is not None:
                layer_hook.after(i)  # every launch that reads this layer's inputs is enqueued
        return {"o_full": o, "lse_full": lse, "scores": None if self.fuse_topk else scores, "idx": idx, "cnt": cnt,
                "layers": outs}

    def forward_from_host(self, q_h, k_h, v_h, layers_h: List[SparseLayerIn], stream=None, fp8_kv=None,
                          intermediates: bool = True, slots: Optional[int] = None):
        """forward() with its inputs in pinned host memory. Q, K and V are copied
        first; every sparse layer's inputs then stream in on a second stream
        while the full layer and the layers before it compute. `slots` device
        copies of a layer's inputs are used in turn (default: one per layer, so
        every copy overlaps the full layer; fewer bound the device memory, a slot
        being refilled once the layer that last used it has run). The outputs
        are device tensors as in forward()."""
        cs = torch.cuda.current_stream(self.device) if stream is None else stream
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream(self.device)
        cp = self._copy_stream
        dev = lambda name, t: None if t is None else self._buf(name, tuple(t.shape), t.dtype)
        q, k, v = dev("h_q", q_h), dev("h_k", k_h), dev("h_v", v_h)
        n_slots = len(layers_h) if slots is None else max(1, min(slots, len(layers_h)))
        slot = [SparseLayerIn(*(dev(f"h_s{j}_{f}", getattr(layers_h[0], f)) for f in ("q", "k_swa", "v_swa",
                                                                                      "gamma")))
                for j in range(n_slots)]
        ready = [torch.cuda.Event() for _ in layers_h]
        done = [torch.cuda.Event() for _ in layers_h]

        def load(i):  # layer i's inputs into slot i % n_slots, on the copy stream
            dst, src = slot[i % n_slots], layers_h[i]
            with torch.cuda.stream(cp):
                for f in ("q", "k_swa", "v_swa", "gamma"):
                    if getattr(src, f) is not None:
                        getattr(dst, f).copy_(getattr(src, f), non_blocking=True)
                ready[i].record(cp)

        cp.wait_stream(cs)  # the previous call is done with these buffers
        with torch.cuda.stream(cp):
            for d_, h_ in ((q, q_h), (k, k_h), (v, v_h)):
                if h_ is not None:
                    d_.copy_(h_, non_blocking=True)
            qkv = torch.cuda.Event()
            qkv.record(cp)
        for i in range(n_slots):
            load(i)
        cs.wait_event(qkv)

        class Hook:
            def before(_, i):
                cs.wait_event(ready[i])
                return slot[i % n_slots]

            def after(_, i):
                done[i].record(cs)
                if i + n_slots < len(layers_h):
                    cp.wait_event(done[i])  # the slot is free once layer i has run
                    load(i + n_slots)

        res = self.forward(q, k, v, [None] * len(layers_h), stream=cs, fp8_kv=fp8_kv, intermediates=intermediates,
                           layer_hook=Hook())
        cs.wait_stream(cp)
        return res

    def launches_per_forward(self, n_layers: int, fp8_prefill: bool = False) -> int:
        """Kernels of this library launched by one forward (memsets excluded):
        full layer 1 (block scores) / 3 (token scores: forward, item prefix,
        score pass) / 1 (decode: both passes in one launch); top-k 1 (none
        when it runs inside the score pass); each
        sparse layer 1 (prefill, with its window branch and gate when fused;
        decode, with its key ranges merged in the same launch), plus 1 for an
        unfused gated SWA branch; an FP8 prefill adds the two expansions, a
        token-level prefill the gather of the selected rows."""
        if self.decode:
            full = 1
        else:
            full = 1 if self.sel.block > 1 else 3
        sparse = 1
        swa = 1 if (self.swa_window > 0 and not (self.fused and not self.decode)) else 0
        gather = 1 if (self.gathered and n_layers > 0) else 0
        topk = 0 if self.fuse_topk else 1
        return full + topk + n_layers * (sparse + swa) + (2 if fp8_prefill else 0) + gather
