#!/usr/bin/env python
"""Benchmark of one hybrid block (1 full layer + N sparse layers) on B200.

Workload (default, the largest single-GPU configuration): agentic ragged
chunked prefill -- 4 sequences with cached contexts {262144, 131072, 65536,
16384} and new chunks {8192, 4096, 8192, 2048} queries, 64 query heads / 1 KV
head, d = 128, token-level top-1024 + forced recent 128, tile 64, 1 full layer
feeding 11 sparse layers; seeded synthetic bf16 N(0,1) inputs with 0.5 %
planted keys. A "step" is one pass of the whole block: hs_full_attn_select
(forward + token-score pass) -> hs_topk_select -> hs_gather_selected_kv
-> 11 x hs_sparse_attn_prefill.
The per-step working set (~5 GB) is larger than the 126 MB L2. On one GPU the
same line also carries a shorter measurement of every other configuration
("workloads"): the block-level HySparse prefill (with its own-cache window
branch and gate fused into each sparse layer), the token-level HySparse2
prefill, decode with bf16 and FP8 KV, and the tiny case.

Multi-GPU (torchrun): one block is partitioned over the ranks
(hybrid_sparse_attention_tma_b200.shard): decode by sequences, GQA prefill by
KV heads (neither has a data-path collective), MQA prefill by contiguous
ranges of selection tiles whose K / V come from one all-gather of every
rank's token shard inside each timed step. value = the block's tokens / the
slowest rank's step time ("strong" scaling: the total work is fixed).

--impl reference: the fp64 CPU oracle on host cores, timed on a bounded
sample of the same workload (one selection tile of 64 queries of the
shortest-context sequence per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "hybrid-block attn tokens/s; TFLOP/s & HBM GB/s as % of roofline (1×B200)"
L2_BYTES = 126 * 1024 * 1024  # B200 L2; the per-kernel timing flushes twice this before each call
KERNEL_SOURCES = ["hybrid_sparse_attention_tma_b200/csrc/attn_fwd.cuh",
                  "hybrid_sparse_attention_tma_b200/csrc/hs_common.cuh"]
# the token-level full layer: the forward, then the score pass with the top-k fused
TOKEN_LAYER_SOURCES = KERNEL_SOURCES + ["hybrid_sparse_attention_tma_b200/csrc/token_scores.cuh",
                                        "hybrid_sparse_attention_tma_b200/csrc/topk.cuh",
                                        "hybrid_sparse_attention_tma_b200/csrc/seqtable.cuh"]
TRAFFIC_SOURCES = {"attn_fwd_full": KERNEL_SOURCES, "full_layer_token": TOKEN_LAYER_SOURCES}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="agentic", choices=list(W.WORKLOADS))
    ap.add_argument("--no-extra", action="store_true",
                    help="measure only --workload (skip the other configurations' short runs)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8-kv", action="store_true",
                    help="FP8-e4m3 KV cache: decode sparse layers read it directly; prefill expands it once per block")
    ap.add_argument("--exclusive", action="store_true",
                    help="window-exclusive top-k: k global tokens drawn before the last query's forced window")
    ap.add_argument("--tokens", type=int, default=0,
                    help="scale a single-sequence workload to this many new tokens (profiling cases)")
    ap.add_argument("--batch", type=int, default=0,
                    help="decode: keep this many of the workload's sequences (profiling cases)")
    return ap.parse_args()


def workload(args) -> W.Workload:
    w = W.WORKLOADS[args.workload]
    if args.tokens and w.batch == 1:
        w = W.scaled(w, ctx=(0,), new=(args.tokens,))
    if args.batch and args.batch < w.batch:
        w = W.scaled(w, ctx=w.ctx[:args.batch], new=w.new[:args.batch])
    if args.exclusive:
        w = w.with_(exclusive=True)
    return w


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained"), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def causal_pairs(w: W.Workload) -> int:
    tot = 0
    for c, n in zip(w.ctx, w.new):
        # queries at positions c..c+n-1 see pos+1 keys
        tot += n * (c + 1) + n * (n - 1) // 2
    return tot


def full_flops(w: W.Workload) -> float:
    return 4.0 * w.head_dim * w.n_q_heads * causal_pairs(w)


def src_hash(kernel: str = "attn_fwd_full") -> str:
    h = hashlib.sha256()
    for p in TRAFFIC_SOURCES[kernel]:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("src_hash") != src_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"hs_clocks_bench_{os.getpid()}.csv")
        self.gpu = gpu_index

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        with open(self.path) as f:
            return summarize_clocks(f)


CLOCK_REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def summarize_clocks(lines):
    """Median SM clock, max clock and the throttle reasons seen in
    `nvidia-smi --query-gpu=index,clocks.sm,clocks.max.sm,power.draw,
    clocks_event_reasons.active,<the four reasons> --format=csv,noheader,nounits`
    lines; None when no line parses."""
    sm, mx, reasons = [], None, set()
    for line in lines:
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 9:
            continue
        try:
            sm.append(float(parts[1]))
            mx = float(parts[2])
        except ValueError:
            continue
        for n, v in zip(CLOCK_REASONS, parts[5:9]):
            if v.lower().startswith("active"):
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def block_seed(w) -> int:
    """Seed of the block's synthetic inputs (the same on every rank)."""
    return 1000 + w.config_index


def rank_problem(w, world: int, rank: int, device, fp8: bool = False):
    """This rank's part of one block (shard.plan): the whole block's inputs are
    drawn from one seed on every rank and sliced. Returns (w_r, inputs_r,
    kv_own): kv_own = (k_shard, v_shard, total_rows, kv_row0, kv_rows) for a
    query-tile shard, whose K / V arrive by all-gather in each step; else
    None. Needles are kept only on one rank."""
    from hybrid_sparse_attention_tma_b200 import shard as S
    full = W.make_block_inputs(w, device=device, seed=block_seed(w))
    if fp8 and full.k_fp8 is None:
        full.k_fp8, full.k_scale = W.quantize_e4m3_per_token(full.k)
        full.v_fp8, full.v_scale = W.quantize_e4m3_per_token(full.v)
    if world == 1:
        return w, full, None
    sh = S.plan(w.ctx, w.new, w.n_q_heads, w.n_kv_heads, w.q_tile, world, w.topk, w.block, w.window,
                w.n_sparse)[rank]
    opt = lambda t, f: None if t is None else f(t).contiguous()  # noqa: E731
    if sh.kind == "kv_heads":
        G = w.group
        hq = slice(sh.kv_head0 * G, (sh.kv_head0 + sh.n_kv_heads) * G)
        hk = slice(sh.kv_head0, sh.kv_head0 + sh.n_kv_heads)
        w_r = w.with_(n_q_heads=sh.n_q_heads, n_kv_heads=sh.n_kv_heads)
        cq, ck = (lambda t: t[:, hq]), (lambda t: t[:, hk])
        layers = [W.LayerInputs(opt(L.q, cq), opt(L.k_swa, ck), opt(L.v_swa, ck), opt(L.gamma, cq))
                  for L in full.layers]
        inp = W.BlockInputs(w_r, opt(full.q, cq), opt(full.k, ck), opt(full.v, ck), layers, full.cu_q, full.cu_kv,
                            [], opt(full.k_fp8, ck), opt(full.v_fp8, ck), opt(full.k_scale, ck),
                            opt(full.v_scale, ck))
        return w_r, inp, None
    w_r = W.scaled(w, ctx=sh.ctx, new=sh.new)
    qs = slice(sh.q_row0, sh.q_row0 + w_r.total_q)
    ks = slice(sh.kv_row0, sh.kv_row0 + sh.kv_rows)
    cq, ck = (lambda t: t[qs]), (lambda t: t[ks])
    layers = [W.LayerInputs(opt(L.q, cq), opt(L.k_swa, ck), opt(L.v_swa, ck), opt(L.gamma, cq)) for L in full.layers]
    cu_q = torch.tensor(w_r.cu_q(), dtype=torch.int32, device=device)
    cu_kv = torch.tensor(w_r.cu_kv(), dtype=torch.int32, device=device)
    inp = W.BlockInputs(w_r, opt(full.q, cq), opt(full.k, ck), opt(full.v, ck), layers, cu_q, cu_kv, [],
                        opt(full.k_fp8, ck), opt(full.v_fp8, ck), opt(full.k_scale, ck), opt(full.v_scale, ck))
    if sh.kind == "batch":
        return w_r, inp, None
    lo, hi = S.token_shard(w.total_kv, rank, world)
    kv_own = (full.k[lo:hi].contiguous(), full.v[lo:hi].contiguous(), w.total_kv, sh.kv_row0, sh.kv_rows)
    return w_r, inp, kv_own


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (every rank gets the result); the
    only collective of the bench, outside the timed region."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(block_tokens: int, ms_per_step: float) -> float:
    """Tokens/s of the whole job: the block's new tokens (all ranks together)
    over the slowest rank's step time."""
    return block_tokens / (ms_per_step / 1e3)


def make_runner(w_r, inp, device):
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200.block import HybridBlock, SparseLayerIn
    vl = hs.Varlen(w_r.cu_q(), w_r.cu_kv(), w_r.n_q_heads, w_r.n_kv_heads, w_r.head_dim, device=device)
    blk = HybridBlock(vl, w_r.q_tile, w_r.block, w_r.topk, w_r.window, w_r.swa_window, device=device,
                      exclusive=w_r.exclusive)
    if blk.decode and w_r.swa_window > 0:  # decode reads each layer's own window cache as a ring
        layers = [SparseLayerIn(L.q, *blk.swa_rings(L.k_swa, L.v_swa), L.gamma) for L in inp.layers]
    else:
        layers = [SparseLayerIn(L.q, L.k_swa, L.v_swa, L.gamma) for L in inp.layers]
    return vl, blk, layers


def visible_counts(w, idx, cnt):
    """sum over (tile, KV head, query) of |V_q| for the sparse layers, from the
    selection actually produced (used for the useful-FLOP and byte counts)."""
    dev = idx.device
    tiles_pos0, tiles_n = [], []
    for a, b, ka, kb in zip(w.cu_q()[:-1], w.cu_q()[1:], w.cu_kv()[:-1], w.cu_kv()[1:]):
        n_b, c_b = b - a, (kb - ka) - (b - a)
        for i in range(0, n_b, w.q_tile):
            tiles_pos0.append(c_b + i)
            tiles_n.append(min(w.q_tile, n_b - i))
    pos0 = torch.tensor(tiles_pos0, device=dev)
    ntq = torch.tensor(tiles_n, device=dev)
    qoff = torch.arange(w.q_tile, device=dev)
    pos = pos0[:, None] + qoff[None, :]                      # [tiles, T]
    qvalid = qoff[None, :] < ntq[:, None]
    k = w.topk
    total = torch.zeros((), dtype=torch.float64, device=dev)
    for g in range(w.n_kv_heads):
        ids = idx[:, g, :k].long()
        valid = torch.arange(k, device=dev)[None, :] < cnt[:, g, None]
        lim = pos - w.window                                 # selected keys must be <= pos - w
        start = ids * w.block                                # block start positions
        # keys of each selected block that are <= lim: clip(lim - start + 1, 0, B)
        per = (lim[:, :, None] - start[:, None, :] + 1).clamp(0, w.block)
        per = per * valid[:, None, :]
        sel = per.sum(-1)
        win = torch.minimum(pos + 1, torch.full_like(pos, w.window)) if w.window > 0 else torch.zeros_like(pos)
        total += ((sel + win) * qvalid).sum().double()
    return float(total)


def distinct_selected_rows(w, idx, cnt):
    """Distinct (token, KV head) rows among all tiles' selected tokens: what a
    gather of the selected rows has to read at least once (neighbouring tiles
    share most of their selections)."""
    dev = idx.device
    tile_seq = []
    for b, (a, e) in enumerate(zip(w.cu_q()[:-1], w.cu_q()[1:])):
        tile_seq += [b] * ((e - a + w.q_tile - 1) // w.q_tile)
    kv0 = torch.tensor(w.cu_kv()[:-1], device=dev)[torch.tensor(tile_seq, device=dev)]
    total = 0
    for g in range(w.n_kv_heads):
        valid = torch.arange(w.topk, device=dev)[None, :] < cnt[:, g, None]
        rows = (kv0[:, None] + idx[:, g, :w.topk].long())[valid]
        total += int(torch.unique(rows).numel())
    return total


def needle_recall(w, inp, idx, cnt):
    """Share of planted keys that the sparse layers see from the query they
    were aimed at: the key lies in that query's forced window, or its block is
    in the top-k set of the query's tile and KV head. Reported overall and for
    keys outside the window (where only the selection can find them)."""
    if not inp.needles:
        return None
    import numpy as np
    last = {}
    for (b, j, p, h) in inp.needles:  # a key planted twice keeps its last aim (as the generator does)
        last[(b, j, h // w.group)] = p
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    tile_base, tb = [], 0
    for n in w.new:
        tile_base.append(tb)
        tb += -(-n // w.q_tile)
    n_all = hit_all = n_out = hit_out = 0
    for (b, j, g), p in last.items():
        c_b = w.kv_lens[b] - w.new[b]
        t = tile_base[b] + (p - c_b) // w.q_tile
        in_win = w.window > 0 and j > p - w.window
        sel = idx_h[t, g, :cnt_h[t, g]]
        in_sel = bool(np.isin(j // w.block, sel))
        n_all += 1
        hit_all += int(in_win or in_sel)
        if not in_win:
            n_out += 1
            hit_out += int(in_sel)
    return {"needles": n_all, "recall": round(hit_all / n_all, 4), "outside_window": n_out,
            "recall_outside_window": round(hit_out / n_out, 4) if n_out else None}


def swa_pairs(w):
    tot = 0
    for c, n in zip(w.ctx, w.new):
        for p_ in range(c, c + n):
            tot += min(p_ + 1, w.swa_window)
    return tot


def bench_ours(args, world, rank, local, w=None, steps=None, with_e2e=True, fp8=None, workload_name=None):
    import torch.distributed as dist
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200 import (full_attn_select, full_attn_select_topk, topk_select,
                                                  sparse_attn_prefill,
                                                  sparse_attn_decode, sparse_swa_gated_prefill,
                                                  gather_selected_kv, swa_gated_decode, HS_KV_BF16,
                                                  HS_KV_FP8_E4M3)
    device = f"cuda:{local}"
    torch.cuda.set_device(local)
    w = workload(args) if w is None else w
    steps = args.steps if steps is None else steps
    fp8 = args.fp8_kv if fp8 is None else fp8
    workload_name = args.workload if workload_name is None else workload_name
    if fp8:
        w = w.with_(fp8_kv=True)
    w_block = w
    w, inp, kv_own = rank_problem(w_block, world, rank, device, fp8)
    vl, blk, layers = make_runner(w, inp, device)
    stream = torch.cuda.current_stream()
    fp8_kv = (inp.k_fp8, inp.v_fp8, inp.k_scale, inp.v_scale) if fp8 else None
    if kv_own is not None:
        # query-tile shard: every step all-gathers the ranks' K / V token shards
        from hybrid_sparse_attention_tma_b200 import shard as S
        k_own, v_own, kv_total, kv_r0, kv_n = kv_own

        def gather_kv():
            kf = S.all_gather_kv(k_own, kv_total)
            vf = S.all_gather_kv(v_own, kv_total)
            return kf[kv_r0:kv_r0 + kv_n], vf[kv_r0:kv_r0 + kv_n]
        inp.k, inp.v = gather_kv()

    for _ in range(max(3, args.warmup)):
        blk.forward(inp.q, inp.k, inp.v, layers, stream=stream, fp8_kv=fp8_kv, intermediates=False)
    torch.cuda.synchronize()
    hs.check_error(blk.ws)
    recall = needle_recall(w, inp, blk._bufs["idx"], blk._bufs["cnt"]) if world == 1 else None

    swa_dec = blk.decode and blk.swa_window > 0
    # with the block's fuse_topk the top-k runs inside the score pass: no top-k launch
    kinds = (["full"] + ([] if blk.fuse_topk else ["topk"]) + ["sparse"] + (["gather"] if blk.gathered else [])
             + (["swa"] if swa_dec else []))
    L0 = layers[0]

    def call(kind, st):
        """One library call of `kind` on stream `st` (the first sparse layer's inputs)."""
        sel, bufs = blk.sel, blk._bufs
        if kind == "full" and blk.fuse_topk:
            full_attn_select_topk(vl, sel, inp.q, inp.k, inp.v, bufs["o_full"], bufs["lse_full"], bufs["scores"],
                                  bufs["idx"], bufs["cnt"], ws=blk.ws, stream=st)
        elif kind == "full":
            full_attn_select(vl, sel, inp.q, inp.k, inp.v, bufs["o_full"], bufs["lse_full"], bufs["scores"],
                             ws=blk.ws, stream=st)
        elif kind == "topk":
            topk_select(vl, sel, bufs["scores"], bufs["idx"], bufs["cnt"], ws=blk.ws, stream=st)
        elif kind == "swa":
            swa_gated_decode(vl, blk.swa_window, L0.q, L0.k_swa, L0.v_swa, L0.gamma, bufs["o_sp0"], bufs["o_l0"],
                             stream=st)
        elif kind == "gather":
            gather_selected_kv(vl, sel, inp.k, inp.v, bufs["idx"], bufs["cnt"], bufs["kg"], bufs["vg"], stream=st)
        elif blk.decode:
            if fp8_kv is not None:
                sparse_attn_decode(vl, sel, L0.q, inp.k_fp8, inp.v_fp8, bufs["idx"], bufs["cnt"], inp.k_scale,
                                   inp.v_scale, HS_KV_FP8_E4M3, o=bufs["o_sp0"], lse=bufs["lse_sp0"], ws=blk.ws,
                                   stream=st)
            else:
                sparse_attn_decode(vl, sel, L0.q, inp.k, inp.v, bufs["idx"], bufs["cnt"], kv_dtype=HS_KV_BF16,
                                   o=bufs["o_sp0"], lse=bufs["lse_sp0"], ws=blk.ws, stream=st)
        elif blk.swa_window > 0:
            # the whole sparse layer: sparse branch, own-cache window, gate
            sparse_swa_gated_prefill(vl, sel, L0.q, inp.k, inp.v, bufs["idx"], bufs["cnt"], blk.swa_window, L0.k_swa,
                                     L0.v_swa, L0.gamma, o=bufs["o_l0"], ws=blk.ws, stream=st)
        else:
            sparse_attn_prefill(vl, sel, L0.q, inp.k, inp.v, bufs["idx"], bufs["cnt"], bufs["o_sp0"],
                                bufs["lse_sp0"], ws=blk.ws, stream=st, kg=bufs.get("kg"), vg=bufs.get("vg"))

    # Launch-bound steps (decode: dozens of microsecond kernels) would time the
    # host's enqueue rate rather than the GPU, so the step and every kernel
    # kind are captured once in CUDA graphs and replayed; the library enqueues
    # only launches and memsets inside a call (its one-time set-up ran during
    # warm-up), so capture is safe.
    # (a step that holds the K / V all-gather runs eagerly: no collective
    # inside a captured graph, and such prefill steps are long)
    step_graph = None
    if kv_own is None:
        step_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(step_graph):
            blk.forward(inp.q, inp.k, inp.v, layers, stream=torch.cuda.current_stream(), fp8_kv=fp8_kv,
                        intermediates=False)

    def eager_step():
        kk, vv = gather_kv()
        blk.forward(inp.q, kk, vv, layers, stream=stream, fp8_kv=fp8_kv, intermediates=False)
    run_step = step_graph.replay if step_graph is not None else eager_step
    # Per-kernel times with a cold L2: every call is preceded by a write of
    # twice the L2 size, and the same flushes alone are timed and subtracted
    # (the sparse decode's gathered rows, ~40 MB, would otherwise stay in L2
    # across back-to-back calls).
    reps = 5
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
    flush_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(flush_graph):
        for _ in range(reps):
            flush.fill_(1)
    kind_graphs = {}
    for kd in kinds:
        gk = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gk):
            for _ in range(reps):
                flush.fill_(1)
                call(kd, torch.cuda.current_stream())
        kind_graphs[kd] = gk
    for _ in range(2):
        run_step()
        flush_graph.replay()
        for gk in kind_graphs.values():
            gk.replay()
    torch.cuda.synchronize()
    hs.check_error(blk.ws)

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local])
                          if os.environ.get("CUDA_VISIBLE_DEVICES") else local)
    clocks.start()
    time.sleep(0.3)
    ms_total = timed(run_step, steps)
    n_kind = max(4, steps // 4)
    ms_flush = timed(flush_graph.replay, n_kind)
    kms = {kd: max(0.0, timed(kind_graphs[kd].replay, n_kind) - ms_flush) / (n_kind * reps) for kd in kinds}
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    hs.check_error(blk.ws)
    vals = max_over_ranks([ms_total] + [kms[kd] for kd in kinds], device)
    ms_total = vals[0]
    kms = {kd: vals[i + 1] for i, kd in enumerate(kinds)}
    ms_step = ms_total / steps
    tokens = w.total_q
    value = whole_job_rate(w_block.total_q, ms_step)

    # ---- algorithmic work of each kernel launch ----
    hbm, tf_burst, tf_sust, src = peaks()
    d, hq, hkv, G = w.head_dim, w.n_q_heads, w.n_kv_heads, w.group
    kv_bytes = w.total_kv * hkv * d * 2
    q_bytes = w.total_q * hq * d * 2
    nblk = (w.max_kv + w.block - 1) // w.block
    n_tiles = w.n_tiles()
    vis = visible_counts(w, blk._bufs["idx"], blk._bufs["cnt"])  # sum_q,g |V_q|
    kernels = {}

    def entry(kind, ms, amount, bound):
        if ms <= 0:
            return
        if bound == "tensor":
            ach = amount / (ms / 1e3) / 1e12
            kernels[kind] = {"bound": "tensor", "ms_per_launch": round(ms, 4), "achieved": round(ach, 1),
                             "unit": "TFLOP/s", "peak": tf_burst, "frac": round(ach / tf_burst, 4),
                             "algorithmic_flop_per_launch": amount}
        else:
            ach = amount / (ms / 1e3) / 1e9
            kernels[kind] = {"bound": "hbm", "ms_per_launch": round(ms, 4), "achieved": round(ach, 1),
                             "unit": "GB/s", "peak": hbm, "frac": round(ach / hbm, 4),
                             "algorithmic_bytes_per_launch": amount}

    if blk.decode:
        # full-layer decode: every K/V row once, Q, O, lse and the token scores
        entry("full", kms["full"], kv_bytes * 2 + q_bytes * 2 + n_tiles * hkv * nblk * 4, "hbm")
        row = d * (1 if fp8 else 2) + (4 if fp8 else 0)
        entry("sparse", kms["sparse"], vis * 2 * row + q_bytes * 2, "hbm")
    else:
        entry("full", kms["full"], full_flops(w), "tensor")
        # a fused layer also runs the own-cache window branch (4 d H_q per
        # visible (query, key) pair of the window)
        swa_flop = 4.0 * d * hq * swa_pairs(w) if w.swa_window > 0 else 0.0
        entry("sparse", kms["sparse"], 4.0 * d * G * vis + swa_flop, "tensor")
    if "topk" in kms:
        entry("topk", kms["topk"], n_tiles * hkv * (nblk * 4 + w.topk * 4), "hbm")
    if blk.gathered:
        # K and V: every (tile, KV head) plane of topk rows written once, the
        # distinct selected rows read once (the rest of the reads hit L2)
        uniq = distinct_selected_rows(w, blk._bufs["idx"], blk._bufs["cnt"])
        entry("gather", kms["gather"], (n_tiles * hkv * w.topk + uniq) * d * 2 * 2, "hbm")
    if swa_dec:
        # the window rows of K and V read from the rings, q, o_sparse and o
        win = sum(min(w.swa_window, kb - ka) for ka, kb in zip(w.cu_kv()[:-1], w.cu_kv()[1:]))
        entry("swa", kms["swa"], win * hkv * d * 2 * 2 + 3 * q_bytes, "hbm")
    per_step = {"full": 1, "topk": 1, "sparse": len(layers), "gather": 1, "swa": len(layers)}
    for kd, e in kernels.items():
        e["share_of_step"] = round(e["ms_per_launch"] * per_step[kd] / ms_step, 4)
    dom = dict(kernels["full"])
    dom["kernel"] = ("full_decode_tc_kernel (both exact passes, one persistent launch)" if blk.decode
                     else "attn_fwd_kernel<d, full, B> (+ token-score pass when B = 1)")
    token_full = w.block == 1 and not blk.decode  # forward + score pass per launch
    dom["traffic"] = traffic_for("full_layer_token" if token_full else "attn_fwd_full", workload_name)
    dom["peak_kind"] = f"{src} {'HBM copy' if blk.decode else 'bf16 burst'}"

    # ---- e2e through the public API with host buffers ----
    e2e = None
    if with_e2e and not args.no_e2e:
        e2e = bench_e2e(args, w, inp, vl, blk, layers, device, w_block.total_q, fp8_kv)

    kind = ("decode" if blk.decode else ("HySparse block-level prefill" if w_block.block > 1 else "HySparse2 token-level prefill"))
    desc = (f"{w_block.name}: {kind}, {w_block.batch}x ctx {list(w_block.ctx)[:4]} + new {list(w_block.new)[:4]} tokens, "
            f"{w_block.n_q_heads}/{w_block.n_kv_heads} heads, d={d}, B={w_block.block}, k={w_block.topk}, w={w_block.window}"
            + (f", SWA {w_block.swa_window}+gate" if w_block.swa_window else "")
            + f", 1 full + {w_block.n_sparse} sparse" + (", FP8-e4m3 KV in the sparse layers" if fp8 else ""))
    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
           "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
           "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded N(0,1) bf16" + (", planted keys)" if w.needle_rate else ")"),
           "config": {"workload": desc, "tokens_per_step": w_block.total_q, "tokens_this_rank": tokens,
                      "l2": "step: inputs larger than L2; per-kernel times: L2 flushed before every call", "parallelism": (f"one block over {world} GPUs: {shard_kind(w_block, world)}" if world > 1
                                      else "one block, one GPU")},
           "roofline": dom, "kernels": kernels,
           "gpu_launches": blk.launches_per_forward(len(layers), fp8_prefill=bool(fp8) and not blk.decode) * steps,
           "needle_recall": recall, "clocks": clk, "e2e": e2e}
    del step_graph, flush_graph, kind_graphs, flush, inp, blk, layers, kv_own
    torch.cuda.empty_cache()
    return out


def shard_kind(w, world):
    from hybrid_sparse_attention_tma_b200 import shard as S
    sh = S.plan(w.ctx, w.new, w.n_q_heads, w.n_kv_heads, w.q_tile, world, w.topk, w.block, w.window, w.n_sparse)
    return {"batch": "sequences per rank", "kv_heads": "KV heads per rank",
            "q_tiles": "selection tiles per rank + K/V all-gather"}[sh[0].kind]


EXTRA = [("hys_block", False), ("hys2_prefill", False), ("decode", False), ("decode", True), ("decode_swa", False),
         ("tiny", False)]


def bench_extra(args, world, rank, local, headline):
    """Short measurements of the other configurations (one GPU only): the
    step rate, the per-kernel roofline entries and the needle recall of each."""
    out = {}
    for name, fp8 in EXTRA:
        if name == headline and not fp8:
            continue
        r = bench_ours(args, world, rank, local, w=W.WORKLOADS[name], steps=max(4, min(args.steps, 10)),
                       with_e2e=False, fp8=fp8, workload_name=name)
        key = name + ("_fp8" if fp8 else "")
        out[key] = {k: r[k] for k in ["value", "unit", "ms_per_step", "steps", "kernels", "needle_recall",
                                      "clocks", "gpu_launches"]}
        out[key]["workload"] = r["config"]["workload"]
    return out


def bench_e2e(args, w, inp, vl, blk, layers, device, block_tokens, fp8_kv=None):
    """Same metric through the block runner's public call with the step's
    inputs in pinned host memory (HybridBlock.forward_from_host: Q, K, V
    copied first, each sparse layer's inputs streamed in on a copy stream
    while the earlier layers compute) and the last layer's output read back."""
    from hybrid_sparse_attention_tma_b200.block import SparseLayerIn
    pin = (lambda t: None if t is None else t.cpu().pin_memory())
    host_q, host_k, host_v = pin(inp.q), pin(inp.k), pin(inp.v)
    hl = [SparseLayerIn(pin(L.q), pin(L.k_swa), pin(L.v_swa), pin(L.gamma)) for L in layers]
    out_host = torch.empty(inp.q.shape, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.current_stream()
    nbytes = (lambda t: 0 if t is None else t.numel() * t.element_size())
    h2d = nbytes(host_q) + nbytes(host_k) + nbytes(host_v)
    h2d += sum(nbytes(getattr(L, f)) for L in hl for f in ("q", "k_swa", "v_swa", "gamma"))
    d2h = out_host.numel() * out_host.element_size()

    def step():
        res = blk.forward_from_host(host_q, host_k, host_v, hl, stream=stream, fp8_kv=fp8_kv, intermediates=False)
        out_host.copy_(res["layers"][-1]["o"], non_blocking=True)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    steps = max(3, args.steps // 4)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    ms = max_over_ranks([ms], device)[0]
    return {"value": round(whole_job_rate(block_tokens, ms), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "steps": steps}


# ---------------------------------------------------------------- oracle side

class _LazyF64:
    """float64 view of a bf16 CPU tensor: only the slices the oracle reads are
    decoded (a whole C5 block in fp64 would take ~18 GB of host memory)."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        import numpy as np
        import oracle as O
        conv = (lambda i: torch.from_numpy(i.astype(np.int64)) if isinstance(i, np.ndarray) else i)
        idx = tuple(conv(i) for i in idx) if isinstance(idx, tuple) else conv(idx)
        return O.bf16_to_f64(W.bf16_bits(self.t[idx]))


def oracle_inputs(inp_cpu):
    """The block's inputs as the oracle reads them (float64 values of the bf16 data)."""
    layers = []
    for L in inp_cpu.layers:
        d = {"q": _LazyF64(L.q)}
        if L.k_swa is not None:
            d.update(k_swa=_LazyF64(L.k_swa), v_swa=_LazyF64(L.v_swa), gamma=L.gamma.double().numpy())
        layers.append(d)
    return _LazyF64(inp_cpu.q), _LazyF64(inp_cpu.k), _LazyF64(inp_cpu.v), layers


def sample_tiles(w):
    """Selection tiles the oracle is timed on: from the middle outwards of the
    sequence with the shortest context (the oracle's cost per query grows with
    the keys it sees, so its rate on these tiles is an upper bound of its rate
    on the whole workload)."""
    import oracle as O
    tiles = O.make_tiles(w.cu_q(), w.cu_kv(), w.q_tile)
    b = min(range(w.batch), key=lambda i: (w.kv_lens[i] if w.new[i] > 0 else 1 << 62))
    own = [t.index for t in tiles if t.seq == b]
    mid = len(own) // 2
    order = [own[mid]]
    for d in range(1, len(own)):
        for j in (mid + d, mid - d):
            if 0 <= j < len(own):
                order.append(own[j])
    return order, tiles


def host_description():
    """CPU model and the number of cores this process may use."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        nproc = len(os.sched_getaffinity(0))
    except Exception:
        nproc = os.cpu_count() or 1
    return {"cpu_model": model, "nproc": nproc}


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def time_oracle(w, n_tiles_sample=1, repeats=1, min_seconds=0.0, max_tiles=8):
    """Time the oracle's whole block on selection tiles of sample_tiles(w), one
    tile per run: `repeats` runs of the first `n_tiles_sample` tiles, or
    (min_seconds > 0) successive tiles until that much oracle time or
    `max_tiles` tiles. Returns (tokens per run, run times)."""
    from oracle.block import run_block
    inp = W.make_block_inputs(w, device="cpu")
    q, k, v, layers = oracle_inputs(inp)
    order, tiles = sample_tiles(w)

    def run(ids):
        t = time.perf_counter()
        run_block(q, k, v, layers, w.cu_q(), w.cu_kv(), w.n_kv_heads, w.q_tile, w.block, w.topk, w.window,
                  w.swa_window, tile_ids=ids, compact=True)
        return time.perf_counter() - t

    if min_seconds > 0:
        toks, times = [], []
        i = 0
        while (sum(times) < min_seconds and i < max_tiles and i < len(order)) or not times:
            tid = order[i % len(order)]
            times.append(run([tid]))
            toks.append(tiles[tid].n)
            i += 1
        return toks, times
    ids = order[:n_tiles_sample]
    toks = sum(tiles[i].n for i in ids)
    return toks, [run(ids) for _ in range(repeats)]


def bench_reference(args, world, rank):
    if rank != 0:
        return None
    w = workload(args)
    import oracle as O  # noqa: F401
    toks, times = time_oracle(w, 1, repeats=args.warmup + args.steps)
    timed = times[args.warmup:]
    s = sum(timed) / len(timed)
    value = toks / s
    cores = oracle_threads()
    order, tiles = sample_tiles(w)
    t0 = tiles[order[0]]
    sample = (f"selection tile {t0.index} of sequence {t0.seq} (its shortest context; {toks} queries at positions "
              f"{t0.pos0}..{t0.last_pos}, all layers of the block) per step; tokens/s extrapolated from it")
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16" + (", planted keys)" if w.needle_rate else ")"),
            "config": {"workload": w.name, "tokens_per_step": toks},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample, "extrapolated": True, **host_description()},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    args = parse()
    world, rank, local = dist_setup()
    if args.impl == "reference":
        out = bench_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out))
        return
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out = bench_ours(args, world, rank, local)
    if world == 1 and not args.no_extra and not args.tokens and not args.batch:
        out["workloads"] = bench_extra(args, world, rank, local, args.workload)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        w = workload(args)
        toks, times = time_oracle(w, min_seconds=10.0)
        out["cpu_baseline"] = {"value": round(sum(toks) / sum(times), 3), "unit": "tokens/s",
                               "cores": oracle_threads(), "kind": "oracle", "extrapolated": True,
                               **host_description(),
                               "sample": f"{len(toks)} selection tiles of the shortest-context sequence "
                                         f"({sum(toks)} queries), whole block, {sum(times):.1f} s; tokens/s "
                                         f"extrapolated from those tiles (an upper bound: longer contexts cost "
                                         f"the oracle more per query)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


if __name__ == "__main__":
    main()
