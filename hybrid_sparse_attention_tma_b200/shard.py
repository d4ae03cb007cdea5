"""Partition of one hybrid block over N GPUs, one process per GPU.

The method's work units are independent once K/V exist: a selection tile's
full-layer rows, scores, top-k and sparse-layer rows depend only on that
tile's queries and the keys before them. So the block shards without any
exchange inside the path:

* decode (one new token per sequence): contiguous ranges of sequences,
  balanced by their key counts; no collective.
* prefill with H_kv a multiple of N (GQA, e.g. 8 KV heads): KV-head groups
  with their query heads; each rank holds its heads' Q / K / V; no collective.
* other prefill (MQA, one KV head): contiguous ranges of selection tiles,
  balanced by an estimate of their cost. A tile needs the keys up to its last
  query, so a rank's queries are one contiguous slice of the packed Q and its
  keys one contiguous slice of the packed K / V (the tail of its first
  sequence's tiles needs that sequence's whole prefix, a middle sequence all
  of it, its last sequence a prefix). Every rank first owns a token shard of
  K / V (as its own projection would produce it) and receives the rest with
  one all-gather (NCCL over NVLink between GPUs; gloo on the CPU tests).

Results stay sharded: rank r writes the rows of its tiles / heads /
sequences. Plain host arithmetic: no kernel and no collective is issued here
except ``all_gather_kv``.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Sequence


@dataclass
class Shard:
    rank: int
    world: int
    kind: str                     # "batch", "kv_heads" or "q_tiles"
    # the rank's sub-problem, in the library's varlen terms
    ctx: List[int] = field(default_factory=list)    # cached keys before the new queries, per sub-sequence
    new: List[int] = field(default_factory=list)    # new queries per sub-sequence
    n_q_heads: int = 0
    n_kv_heads: int = 0
    # where it sits in the whole block
    seqs: List[int] = field(default_factory=list)   # original sequence of each sub-sequence
    kv_head0: int = 0                               # first KV head (kv_heads sharding)
    tile0: int = 0                                  # first global selection tile (q_tiles / batch)
    n_tiles: int = 0
    q_row0: int = 0                                 # first packed query row of the slice
    kv_row0: int = 0                                # first packed key row of the slice
    kv_rows: int = 0                                # packed key rows of the slice


def _prefix(xs):
    out = [0]
    for x in xs:
        out.append(out[-1] + x)
    return out


def _balanced_cuts(costs: Sequence[float], world: int) -> List[int]:
    """Contiguous split of len(costs) items into `world` ranges of about equal
    total cost: boundaries[r] .. boundaries[r + 1] for rank r."""
    pre = _prefix(costs)
    total = pre[-1]
    cuts = [0]
    j = 0
    for r in range(1, world):
        target = total * r / world
        while j < len(costs) and pre[j + 1] <= target:
            j += 1
        # take item j if that brings the prefix closer to the target
        if j < len(costs) and pre[j + 1] - target < target - pre[j]:
            j += 1
        cuts.append(max(cuts[-1], j))
    cuts.append(len(costs))
    return cuts


def tile_costs(ctx, new, T: int, n_q_heads: int, topk: int, block: int, window: int, n_sparse: int):
    """Estimated cost of every selection tile, in (query, key) pairs: the full
    layer's causal pairs of its queries plus n_sparse times its queries'
    sparse sets (k blocks + window), all times the query heads."""
    out = []
    for c, n in zip(ctx, new):
        for i in range(0, n, T):
            m = min(T, n - i)
            p0 = c + i
            full = m * (p0 + 1) + m * (m - 1) // 2
            sparse = m * min(p0 + m, topk * block + window) * n_sparse
            out.append(float(full + sparse) * n_q_heads)
    return out


def plan(ctx: Sequence[int], new: Sequence[int], n_q_heads: int, n_kv_heads: int, T: int, world: int,
         topk: int = 0, block: int = 1, window: int = 0, n_sparse: int = 0) -> List[Shard]:
    """Per-rank shards of one block (see the module docstring for the rules)."""
    ctx, new = list(ctx), list(new)
    B = len(new)
    kv = [c + n for c, n in zip(ctx, new)]
    cu_q, cu_kv = _prefix(new), _prefix(kv)
    tiles_per_seq = [-(-n // T) for n in new]
    tile_base = _prefix(tiles_per_seq)
    shards: List[Shard] = []
    if all(n == 1 for n in new):
        cuts = _balanced_cuts([float(x) for x in kv], world)
        for r in range(world):
            b0, b1 = cuts[r], cuts[r + 1]
            shards.append(Shard(r, world, "batch", ctx[b0:b1], new[b0:b1], n_q_heads, n_kv_heads,
                                list(range(b0, b1)), 0, tile_base[b0], tile_base[b1] - tile_base[b0],
                                cu_q[b0], cu_kv[b0], cu_kv[b1] - cu_kv[b0]))
        return shards
    if n_kv_heads % world == 0:
        per = n_kv_heads // world
        G = n_q_heads // n_kv_heads
        for r in range(world):
            shards.append(Shard(r, world, "kv_heads", ctx, new, per * G, per, list(range(B)), r * per, 0,
                                tile_base[B], 0, 0, cu_kv[B]))
        return shards
    # contiguous selection tiles, balanced by cost
    costs = tile_costs(ctx, new, T, n_q_heads, topk, block, window, n_sparse)
    cuts = _balanced_cuts(costs, world)
    for r in range(world):
        t0, t1 = cuts[r], cuts[r + 1]
        sh = Shard(r, world, "q_tiles", n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, tile0=t0, n_tiles=t1 - t0)
        if t1 > t0:
            b_first = max(b for b in range(B) if tile_base[b] <= t0 and tiles_per_seq[b] > 0)
            b_last = max(b for b in range(B) if tile_base[b] <= t1 - 1 and tiles_per_seq[b] > 0)
            for b in range(b_first, b_last + 1):
                i0 = (t0 - tile_base[b]) if b == b_first else 0
                i1 = (t1 - tile_base[b]) if b == b_last else tiles_per_seq[b]
                q_lo, q_hi = i0 * T, min(i1 * T, new[b])
                if q_hi <= q_lo:
                    continue
                sh.seqs.append(b)
                sh.ctx.append(ctx[b] + q_lo)
                sh.new.append(q_hi - q_lo)
            b0 = sh.seqs[0]
            sh.q_row0 = cu_q[b0] + (t0 - tile_base[b0]) * T
            sh.kv_row0 = cu_kv[b0]
            last = sh.seqs[-1]
            sh.kv_rows = cu_kv[last] + sh.ctx[-1] + sh.new[-1] - cu_kv[b0]
        shards.append(sh)
    return shards


def token_shard(total_rows: int, rank: int, world: int):
    """Rows [lo, hi) of a packed K / V tensor that rank `rank` owns before the
    all-gather (equal contiguous shards; the last may be shorter)."""
    per = -(-total_rows // world)
    lo = min(total_rows, rank * per)
    return lo, min(total_rows, lo + per)


def all_gather_kv(shard_rows, total_rows: int, group=None):
    """Every rank's token shard of a [rows, H_kv, d] tensor -> the whole tensor
    on every rank (one all-gather; shards padded to equal length)."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    per = -(-total_rows // world)
    pad = torch.zeros((per,) + tuple(shard_rows.shape[1:]), dtype=shard_rows.dtype, device=shard_rows.device)
    pad[:shard_rows.shape[0]] = shard_rows
    if dist.get_backend(group) == "nccl":
        out = torch.empty((per * world,) + tuple(shard_rows.shape[1:]), dtype=shard_rows.dtype,
                          device=shard_rows.device)
        dist.all_gather_into_tensor(out, pad, group=group)
    else:
        parts = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(parts, pad, group=group)
        out = torch.cat(parts, 0)
    return out[:total_rows]
