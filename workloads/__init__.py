"""Seeded synthetic inputs for the hybrid-block attention path.

This module is shared by the fp64 oracle tests and the CUDA path. It only
draws random numbers and lays them out; it contains none of the method's
arithmetic (no softmax, no scores, no selection).

Workload shapes follow the five hybrid-block configurations:

* ``tiny``        -- 1 x 512 causal tokens, 4 query heads on 1 KV head, d=64,
                     16-token blocks, top-8 blocks + forced window 32, tile 16.
* ``hys_block``   -- HySparse block-level prefill: 32768 tokens, 32/8 heads,
                     d=128, 64-token blocks, top-16, separate SWA window 128
                     merged by a sigmoid gate, 3 sparse layers, 1 % planted keys.
* ``hys2_prefill``-- HySparse2 token-level prefill: 65536 tokens, 64/1 heads,
                     top-1024 tokens + forced 128, tile 64, 11 sparse layers,
                     0.5 % planted keys.
* ``decode``      -- 64 sequences x 131072 cached tokens, one new query each,
                     64/1 heads, top-1024 + forced 128, bf16 or FP8-e4m3 KV.
* ``agentic``     -- ragged chunked prefill: contexts {262144, 131072, 65536,
                     16384} + new chunks {8192, 4096, 8192, 2048}, 64/1 heads.

Planted keys ("needles"): for a fraction rho of key positions j of each
sequence, a query position p >= j (among that sequence's new queries) and a
head h of the KV head's group are drawn uniformly, and the key row is set to
4 * sqrt(d) * Q[p, h] / ||Q[p, h]||, i.e. four times the typical key norm,
pointing at that query.

FP8 KV inputs are produced by a plain per-token quantiser (one fp32 scale per
token and KV head, scale = max|x| / 448, codes = round-to-nearest-even of
x / scale, saturated to +-448). The quantiser is input preparation: the
decode kernels and the oracle both receive the codes and the scales.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import torch

FP8_E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    ctx: tuple            # cached context per sequence (tokens before the new chunk)
    new: tuple            # new query tokens per sequence
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    q_tile: int           # T: queries per selection tile
    block: int            # B: keys per selectable block (1 = token level)
    topk: int             # k, in blocks
    window: int           # w: forced recent window inside the sparse set
    n_sparse: int         # sparse layers fed by the one full layer
    swa_window: int = 0   # >0: separate SWA branch with its own KV + sigmoid gate
    needle_rate: float = 0.0
    fp8_kv: bool = False  # decode only: KV cache given as e4m3 codes + scales
    config_index: int = 0
    exclusive: bool = False  # top-k drawn only from blocks before the last query's forced window

    @property
    def batch(self) -> int:
        return len(self.new)

    @property
    def kv_lens(self) -> List[int]:
        return [c + n for c, n in zip(self.ctx, self.new)]

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def total_q(self) -> int:
        return sum(self.new)

    @property
    def total_kv(self) -> int:
        return sum(self.kv_lens)

    @property
    def max_q(self) -> int:
        return max(self.new)

    @property
    def max_kv(self) -> int:
        return max(self.kv_lens)

    def cu_q(self) -> List[int]:
        out = [0]
        for n in self.new:
            out.append(out[-1] + n)
        return out

    def cu_kv(self) -> List[int]:
        out = [0]
        for n in self.kv_lens:
            out.append(out[-1] + n)
        return out

    def n_tiles(self) -> int:
        return sum((n + self.q_tile - 1) // self.q_tile for n in self.new)

    def n_blocks_max(self) -> int:
        return (self.max_kv + self.block - 1) // self.block

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", ctx=(0,), new=(512,), n_q_heads=4, n_kv_heads=1, head_dim=64,
                     q_tile=16, block=16, topk=8, window=32, n_sparse=1, config_index=0),
    "hys_block": Workload("hys_block", ctx=(0,), new=(32768,), n_q_heads=32, n_kv_heads=8,
                          head_dim=128, q_tile=64, block=64, topk=16, window=0, n_sparse=3,
                          swa_window=128, needle_rate=0.01, config_index=1),
    "hys2_prefill": Workload("hys2_prefill", ctx=(0,), new=(65536,), n_q_heads=64, n_kv_heads=1,
                             head_dim=128, q_tile=64, block=1, topk=1024, window=128, n_sparse=11,
                             needle_rate=0.005, config_index=2),
    "decode": Workload("decode", ctx=(131071,) * 64, new=(1,) * 64, n_q_heads=64, n_kv_heads=1,
                       head_dim=128, q_tile=1, block=1, topk=1024, window=128, n_sparse=11,
                       config_index=3),
    # the HySparse layer shape (C2) at decode time: 64-token blocks, top-16, own
    # 128-token window kept as a ring + sigmoid gate; 64 sequences x 32k cached tokens
    "decode_swa": Workload("decode_swa", ctx=(32767,) * 64, new=(1,) * 64, n_q_heads=32, n_kv_heads=8,
                           head_dim=128, q_tile=1, block=64, topk=16, window=0, n_sparse=3, swa_window=128,
                           config_index=1),
    "agentic": Workload("agentic", ctx=(262144, 131072, 65536, 16384), new=(8192, 4096, 8192, 2048),
                        n_q_heads=64, n_kv_heads=1, head_dim=128, q_tile=64, block=1, topk=1024,
                        window=128, n_sparse=11, needle_rate=0.005, config_index=4),
}


def scaled(w: Workload, *, ctx=None, new=None, **kw) -> Workload:
    """A smaller copy of a workload (same head layout and selection rule)."""
    return w.with_(ctx=tuple(ctx) if ctx is not None else w.ctx,
                   new=tuple(new) if new is not None else w.new, **kw)


@dataclasses.dataclass
class LayerInputs:
    q: torch.Tensor                    # [T_q, H_q, d] bf16
    k_swa: Optional[torch.Tensor]      # [T_kv, H_kv, d] bf16 (HySparse SWA branch)
    v_swa: Optional[torch.Tensor]
    gamma: Optional[torch.Tensor]      # [T_q, H_q] fp32 gate logits


@dataclasses.dataclass
class BlockInputs:
    w: Workload
    q: torch.Tensor                    # full layer Q [T_q, H_q, d] bf16
    k: torch.Tensor                    # shared KV cache [T_kv, H_kv, d] bf16
    v: torch.Tensor
    layers: List[LayerInputs]
    cu_q: torch.Tensor                 # int32 [batch+1]
    cu_kv: torch.Tensor                # int32 [batch+1]
    needles: List[tuple]               # (seq, key position, query position, head)
    k_fp8: Optional[torch.Tensor] = None   # uint8 e4m3 codes [T_kv, H_kv, d]
    v_fp8: Optional[torch.Tensor] = None
    k_scale: Optional[torch.Tensor] = None  # fp32 [T_kv, H_kv]
    v_scale: Optional[torch.Tensor] = None


def _normal_bf16(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-(token, KV head) FP8-e4m3 quantiser used to prepare FP8 KV inputs.

    x: [T, H, d] (any float dtype). Returns (codes uint8 [T, H, d], scale fp32 [T, H]).
    scale = max|x| / 448 (1 where the row is all zero); codes = e4m3(x / scale)
    rounded to nearest even and saturated to +-448.
    """
    xf = x.float()
    amax = xf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / FP8_E4M3_MAX, torch.ones_like(amax))
    y = (xf / scale.unsqueeze(-1)).clamp(-FP8_E4M3_MAX, FP8_E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()


def make_block_inputs(w: Workload, device="cpu", seed: Optional[int] = None,
                      n_sparse: Optional[int] = None) -> BlockInputs:
    """Draw one hybrid block's inputs.

    Draw order (one torch.Generator, seed 1000 + config index unless given):
    Q_full, K, V, then per sparse layer (Q_l[, K_swa_l, V_swa_l, gamma_l]),
    then the needle plan.
    """
    if seed is None:
        seed = 1000 + w.config_index
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    d, hq, hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
    tq, tkv = w.total_q, w.total_kv
    q = _normal_bf16((tq, hq, d), gen, device)
    k = _normal_bf16((tkv, hkv, d), gen, device)
    v = _normal_bf16((tkv, hkv, d), gen, device)
    layers = []
    for _ in range(w.n_sparse if n_sparse is None else n_sparse):
        ql = _normal_bf16((tq, hq, d), gen, device)
        if w.swa_window > 0:
            ks = _normal_bf16((tkv, hkv, d), gen, device)
            vs = _normal_bf16((tkv, hkv, d), gen, device)
            gm = torch.randn((tq, hq), generator=gen, device=device, dtype=torch.float32)
            layers.append(LayerInputs(ql, ks, vs, gm))
        else:
            layers.append(LayerInputs(ql, None, None, None))
    needles = []
    if w.needle_rate > 0:
        cu_q, cu_kv = w.cu_q(), w.cu_kv()
        for b in range(w.batch):
            kv_b, n_b = w.kv_lens[b], w.new[b]
            c_b = kv_b - n_b
            n_needles = int(math.floor(w.needle_rate * kv_b))
            if n_needles == 0:
                continue
            js = torch.randint(0, kv_b, (n_needles,), generator=gen, device=device).tolist()
            us = torch.rand((n_needles, 3), generator=gen, device=device, dtype=torch.float64).tolist()
            for j, (u0, u1, u2) in zip(js, us):
                lo = max(j, c_b)
                p = lo + min(int(u0 * (kv_b - lo)), kv_b - lo - 1)
                g = min(int(u2 * hkv), hkv - 1)
                h = g * w.group + min(int(u1 * w.group), w.group - 1)
                needles.append((b, j, p, h))
        # K[j, g] <- 4 sqrt(d) Q[p, h] / ||Q[p, h]||; a key drawn twice keeps its last plan
        last = {}
        for (b, j, p, h) in needles:
            last[(b, j, h // w.group)] = (p, h)
        if last:
            keys = list(last.keys())
            rows_q = torch.tensor([cu_q[b] + (last[(b, j, g)][0] - (w.kv_lens[b] - w.new[b]))
                                   for (b, j, g) in keys], device=device)
            heads = torch.tensor([last[key][1] for key in keys], device=device)
            rows_k = torch.tensor([cu_kv[b] + j for (b, j, g) in keys], device=device)
            gs = torch.tensor([g for (b, j, g) in keys], device=device)
            qv = q[rows_q, heads].float()
            kn = 4.0 * math.sqrt(d) * qv / qv.norm(dim=-1, keepdim=True)
            k[rows_k, gs] = kn.to(torch.bfloat16)
    cu_q_t = torch.tensor(w.cu_q(), dtype=torch.int32, device=device)
    cu_kv_t = torch.tensor(w.cu_kv(), dtype=torch.int32, device=device)
    out = BlockInputs(w, q, k, v, layers, cu_q_t, cu_kv_t, needles)
    if w.fp8_kv:
        out.k_fp8, out.k_scale = quantize_e4m3_per_token(k)
        out.v_fp8, out.v_scale = quantize_e4m3_per_token(v)
    return out


def bf16_bits(x: torch.Tensor):
    """Raw bf16 bit patterns of a tensor, as a numpy uint16 array on the host."""
    return x.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
