#!/usr/bin/env python
"""Benchmark of one hybrid block (1 full layer + N sparse layers) on B200.

Workload (default): HySparse block-level prefill, 1 x 32768 tokens, 32 query
heads / 8 KV heads, d = 128, 64-token blocks, top-16, separate SWA window 128
+ sigmoid gate, 1 full layer feeding 3 sparse layers; seeded synthetic bf16
N(0,1) inputs with 1 % planted keys. A "step" is one pass of the whole block:
hs_full_attn_select -> hs_topk_select -> 3 x hs_sparse_swa_gated_prefill (the
sparse branch, the own-cache window branch and the gate of one layer in one
launch). The per-step working set (~2 GB) is larger than the 126 MB L2.

Multi-GPU (torchrun): every rank runs its own independent block (its own
sequences); no data-path collective. value = tokens of all ranks / max-over-
ranks time ("weak" scaling).

--impl reference: the fp64 CPU oracle on host cores, timed on a bounded
sample of the same workload (one selection tile of 64 queries per step).
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="hys_block", choices=list(W.WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--fp8-kv", action="store_true", help="decode: sparse layers read an FP8-e4m3 KV cache")
    ap.add_argument("--tokens", type=int, default=0,
                    help="scale a single-sequence workload to this many new tokens (profiling cases)")
    return ap.parse_args()


def workload(args) -> W.Workload:
    w = W.WORKLOADS[args.workload]
    if args.tokens and w.batch == 1:
        w = W.scaled(w, ctx=(0,), new=(args.tokens,))
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


def src_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
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
    if not e or e.get("src_hash") != src_hash():
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


def rank_seed(w, rank: int) -> int:
    """Seed of the independent block rank `rank` processes (distinct per rank)."""
    return 1000 + w.config_index + 7919 * rank


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (every rank gets the result); the
    only collective of the bench, outside the timed region."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Tokens/s of the whole job: every rank's tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def make_runner(w, device, seed):
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200.block import HybridBlock, SparseLayerIn
    inp = W.make_block_inputs(w, device=device, seed=seed)
    vl = hs.Varlen(w.cu_q(), w.cu_kv(), w.n_q_heads, w.n_kv_heads, w.head_dim, device=device)
    blk = HybridBlock(vl, w.q_tile, w.block, w.topk, w.window, w.swa_window, device=device)
    layers = [SparseLayerIn(L.q, L.k_swa, L.v_swa, L.gamma) for L in inp.layers]
    return inp, vl, blk, layers


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


def swa_pairs(w):
    tot = 0
    for c, n in zip(w.ctx, w.new):
        for p_ in range(c, c + n):
            tot += min(p_ + 1, w.swa_window)
    return tot


def bench_ours(args, world, rank, local):
    import torch.distributed as dist
    import hybrid_sparse_attention_tma_b200 as hs
    from hybrid_sparse_attention_tma_b200 import (full_attn_select, topk_select, sparse_attn_prefill,
                                                  sparse_attn_decode, sparse_swa_gated_prefill, HS_KV_BF16,
                                                  HS_KV_FP8_E4M3)
    device = f"cuda:{local}"
    torch.cuda.set_device(local)
    w = workload(args)
    if args.fp8_kv:
        w = w.with_(fp8_kv=True)
    inp, vl, blk, layers = make_runner(w, device, seed=rank_seed(w, rank))
    stream = torch.cuda.current_stream()
    fp8_kv = (inp.k_fp8, inp.v_fp8, inp.k_scale, inp.v_scale) if args.fp8_kv else None

    for _ in range(max(3, args.warmup)):
        blk.forward(inp.q, inp.k, inp.v, layers, stream=stream, fp8_kv=fp8_kv, intermediates=False)
    torch.cuda.synchronize()
    hs.check_error(blk.ws)

    kinds = ["full", "topk", "sparse"]
    L0 = layers[0]

    def call(kind, st):
        """One library call of `kind` on stream `st` (the first sparse layer's inputs)."""
        sel, bufs = blk.sel, blk._bufs
        if kind == "full":
            full_attn_select(vl, sel, inp.q, inp.k, inp.v, bufs["o_full"], bufs["lse_full"], bufs["scores"],
                             ws=blk.ws, stream=st)
        elif kind == "topk":
            topk_select(vl, sel, bufs["scores"], bufs["idx"], bufs["cnt"], ws=blk.ws, stream=st)
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
                                bufs["lse_sp0"], ws=blk.ws, stream=st)

    # Launch-bound steps (decode: dozens of microsecond kernels) would time the
    # host's enqueue rate rather than the GPU, so the step and every kernel
    # kind are captured once in CUDA graphs and replayed; the library enqueues
    # only launches and memsets inside a call (its one-time set-up ran during
    # warm-up), so capture is safe.
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph):
        blk.forward(inp.q, inp.k, inp.v, layers, stream=torch.cuda.current_stream(), fp8_kv=fp8_kv,
                    intermediates=False)
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
        step_graph.replay()
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
    ms_total = timed(step_graph.replay, args.steps)
    n_kind = max(4, args.steps // 4)
    ms_flush = timed(flush_graph.replay, n_kind)
    kms = {kd: max(0.0, timed(kind_graphs[kd].replay, n_kind) - ms_flush) / (n_kind * reps) for kd in kinds}
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    hs.check_error(blk.ws)
    vals = max_over_ranks([ms_total] + [kms[kd] for kd in kinds], device)
    ms_total = vals[0]
    kms = {kd: vals[i + 1] for i, kd in enumerate(kinds)}
    ms_step = ms_total / args.steps
    tokens = w.total_q
    value = whole_job_rate(world, tokens, ms_step)

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
        row = d * (1 if args.fp8_kv else 2) + (4 if args.fp8_kv else 0)
        entry("sparse", kms["sparse"], vis * 2 * row + q_bytes * 2, "hbm")
    else:
        entry("full", kms["full"], full_flops(w), "tensor")
        # a fused layer also runs the own-cache window branch (4 d H_q per
        # visible (query, key) pair of the window)
        swa_flop = 4.0 * d * hq * swa_pairs(w) if w.swa_window > 0 else 0.0
        entry("sparse", kms["sparse"], 4.0 * d * G * vis + swa_flop, "tensor")
    entry("topk", kms["topk"], n_tiles * hkv * (nblk * 4 + w.topk * 4), "hbm")
    per_step = {"full": 1, "topk": 1, "sparse": len(layers)}
    for kd, e in kernels.items():
        e["share_of_step"] = round(e["ms_per_launch"] * per_step[kd] / ms_step, 4)
    dom = dict(kernels["full"])
    dom["kernel"] = ("full-layer decode (two split-K passes + combines)" if blk.decode
                     else "attn_fwd_kernel<d, full, B> (+ token-score pass when B = 1)")
    dom["traffic"] = traffic_for("attn_fwd_full", args.workload)
    dom["peak_kind"] = f"{src} {'HBM copy' if blk.decode else 'bf16 burst'}"

    # ---- e2e through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = bench_e2e(args, w, inp, vl, blk, layers, device, world, fp8_kv)

    kind = ("decode" if blk.decode else ("HySparse block-level prefill" if w.block > 1 else "HySparse2 token-level prefill"))
    desc = (f"{w.name}: {kind}, {w.batch}x ctx {list(w.ctx)[:4]} + new {list(w.new)[:4]} tokens, "
            f"{hq}/{hkv} heads, d={d}, B={w.block}, k={w.topk}, w={w.window}"
            + (f", SWA {w.swa_window}+gate" if w.swa_window else "")
            + f", 1 full + {w.n_sparse} sparse" + (", FP8-e4m3 KV in the sparse layers" if args.fp8_kv else ""))
    out = {"metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic (seeded N(0,1) bf16" + (", planted keys)" if w.needle_rate else ")"),
           "config": {"workload": desc, "tokens_per_step_per_gpu": tokens,
                      "l2": "step: inputs larger than L2; per-kernel times: L2 flushed before every call", "parallelism": f"independent blocks x{world}"},
           "roofline": dom, "kernels": kernels,
           "gpu_launches": blk.launches_per_forward(len(layers)) * args.steps,
           "clocks": clk, "e2e": e2e}
    return out


def bench_e2e(args, w, inp, vl, blk, layers, device, world, fp8_kv=None):
    """Same metric through HybridBlock.forward with the step's inputs copied
    from pinned host memory each step and the last layer's output read back."""
    from hybrid_sparse_attention_tma_b200.block import SparseLayerIn
    host = {"q": inp.q.cpu().pin_memory(), "k": inp.k.cpu().pin_memory(), "v": inp.v.cpu().pin_memory()}
    hl = []
    for L in inp.layers:
        d = {"q": L.q.cpu().pin_memory()}
        if L.k_swa is not None:
            d.update(k_swa=L.k_swa.cpu().pin_memory(), v_swa=L.v_swa.cpu().pin_memory(),
                     gamma=L.gamma.cpu().pin_memory())
        hl.append(d)
    dev_q, dev_k, dev_v = torch.empty_like(inp.q), torch.empty_like(inp.k), torch.empty_like(inp.v)
    dev_layers = [SparseLayerIn(torch.empty_like(L.q),
                                torch.empty_like(L.k_swa) if L.k_swa is not None else None,
                                torch.empty_like(L.v_swa) if L.v_swa is not None else None,
                                torch.empty_like(L.gamma) if L.gamma is not None else None) for L in inp.layers]
    out_host = torch.empty(inp.q.shape, dtype=torch.bfloat16).pin_memory()
    stream = torch.cuda.current_stream()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    h2d += sum(t.numel() * t.element_size() for d in hl for t in d.values())
    d2h = out_host.numel() * out_host.element_size()

    def step():
        dev_q.copy_(host["q"], non_blocking=True)
        dev_k.copy_(host["k"], non_blocking=True)
        dev_v.copy_(host["v"], non_blocking=True)
        for dl, d in zip(dev_layers, hl):
            dl.q.copy_(d["q"], non_blocking=True)
            if dl.k_swa is not None:
                dl.k_swa.copy_(d["k_swa"], non_blocking=True)
                dl.v_swa.copy_(d["v_swa"], non_blocking=True)
                dl.gamma.copy_(d["gamma"], non_blocking=True)
        res = blk.forward(dev_q, dev_k, dev_v, dev_layers, stream=stream, fp8_kv=fp8_kv, intermediates=False)
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
    return {"value": round(whole_job_rate(world, w.total_q, ms), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 3), "steps": steps}


# ---------------------------------------------------------------- oracle side

def oracle_sample(w, tile_id, inp_cpu):
    """Run the oracle's whole block on one selection tile; returns tokens."""
    import numpy as np
    import oracle as O
    from oracle.block import run_block
    q = O.bf16_to_f64(W.bf16_bits(inp_cpu.q))
    k = O.bf16_to_f64(W.bf16_bits(inp_cpu.k))
    v = O.bf16_to_f64(W.bf16_bits(inp_cpu.v))
    layers = []
    for L in inp_cpu.layers:
        d = {"q": O.bf16_to_f64(W.bf16_bits(L.q))}
        if L.k_swa is not None:
            d.update(k_swa=O.bf16_to_f64(W.bf16_bits(L.k_swa)), v_swa=O.bf16_to_f64(W.bf16_bits(L.v_swa)),
                     gamma=L.gamma.double().numpy())
        layers.append(d)
    return q, k, v, layers


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def time_oracle(w, n_tiles_sample=1, repeats=1, min_seconds=0.0, max_tiles=8):
    """Time the oracle's whole block on middle selection tiles, one tile per
    run: `repeats` runs of the first `n_tiles_sample` tiles, or (min_seconds >
    0) successive tiles until that much oracle time or `max_tiles` tiles.
    Returns (tokens per run, run times)."""
    import oracle as O
    from oracle.block import run_block
    inp = W.make_block_inputs(w, device="cpu")
    q, k, v, layers = oracle_sample(w, 0, inp)
    n_t = w.n_tiles()
    tiles = O.make_tiles(w.cu_q(), w.cu_kv(), w.q_tile)

    def run(ids):
        t = time.perf_counter()
        run_block(q, k, v, layers, w.cu_q(), w.cu_kv(), w.n_kv_heads, w.q_tile, w.block, w.topk, w.window,
                  w.swa_window, tile_ids=ids)
        return time.perf_counter() - t

    if min_seconds > 0:
        toks, times = [], []
        i = 0
        while (sum(times) < min_seconds and i < max_tiles) or not times:
            tid = min(n_t - 1, n_t // 2 + i)
            times.append(run([tid]))
            toks.append(tiles[tid].n)
            i += 1
        return toks, times
    mids = [min(n_t - 1, n_t // 2 + i) for i in range(n_tiles_sample)]
    toks = sum(tiles[i].n for i in mids)
    return toks, [run(mids) for _ in range(repeats)]


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
    sample = f"selection tile {w.n_tiles() // 2} ({toks} queries, all layers of the block) per step"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(s * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) bf16, 1% planted keys)",
            "config": {"workload": w.name, "tokens_per_step": toks},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
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
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        w = workload(args)
        toks, times = time_oracle(w, min_seconds=10.0)
        out["cpu_baseline"] = {"value": round(sum(toks) / sum(times), 3), "unit": "tokens/s",
                               "cores": oracle_threads(), "kind": "oracle",
                               "sample": f"{len(toks)} middle selection tiles ({sum(toks)} queries), whole block, "
                                         f"{sum(times):.1f} s"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


if __name__ == "__main__":
    main()
