"""Partition of one hybrid block over N GPUs (host logic, CPU).

* Every configuration's shards at N = 2, 3, 4, 8 cover each sequence, KV head
  or selection tile exactly once, in contiguous packed slices, with the
  query-tile shards balanced by their estimated cost.
* The fp64 oracle run on each rank's sub-problem (its slice of Q and of the
  packed K / V) gives exactly the whole block's rows for those tiles: full
  layer, scores, top-k and sparse layers.
* Two gloo ranks all-gather their K / V token shards into the whole tensor.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import workloads as W
from oracle.block import run_block, tile_rows
from hybrid_sparse_attention_tma_b200 import shard as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _plan(w, world):
    return S.plan(w.ctx, w.new, w.n_q_heads, w.n_kv_heads, w.q_tile, world, w.topk, w.block, w.window, w.n_sparse)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
@pytest.mark.parametrize("world", [2, 3, 4, 8])
def test_shards_cover_the_block_once(name, world):
    w = W.WORKLOADS[name]
    shards = _plan(w, world)
    assert [s.rank for s in shards] == list(range(world))
    kinds = {s.kind for s in shards}
    assert len(kinds) == 1
    kind = kinds.pop()
    if all(n == 1 for n in w.new):
        assert kind == "batch"
        seqs = [b for s in shards for b in s.seqs]
        assert seqs == list(range(w.batch))  # every sequence once, in order
        for s in shards:
            assert list(s.ctx) == [w.ctx[b] for b in s.seqs] and list(s.new) == [w.new[b] for b in s.seqs]
    elif w.n_kv_heads % world == 0:
        assert kind == "kv_heads"
        heads = [g for s in shards for g in range(s.kv_head0, s.kv_head0 + s.n_kv_heads)]
        assert heads == list(range(w.n_kv_heads))
        assert all(s.n_q_heads == s.n_kv_heads * w.group for s in shards)
    else:
        assert kind == "q_tiles"
        tiles = O.make_tiles(w.cu_q(), w.cu_kv(), w.q_tile)
        got = []
        for s in shards:
            got.extend(range(s.tile0, s.tile0 + s.n_tiles))
            if s.n_tiles == 0:
                continue
            # the sub-problem's tiles are the block's tiles, position for position
            sub = O.make_tiles(W.scaled(w, ctx=s.ctx, new=s.new).cu_q(), W.scaled(w, ctx=s.ctx, new=s.new).cu_kv(),
                               w.q_tile)
            assert len(sub) == s.n_tiles
            for a, t in zip(sub, tiles[s.tile0:s.tile0 + s.n_tiles]):
                assert (a.pos0, a.n) == (t.pos0, t.n)
                assert a.row0 + s.q_row0 == t.row0                      # contiguous query slice
                assert a.kv0 + s.kv_row0 == t.kv0                        # keys of the same sequence
                assert a.kv_len >= t.last_pos + 1                        # every key the tile needs
            assert s.kv_row0 + s.kv_rows <= w.total_kv
        assert got == list(range(len(tiles)))
        # balance: no rank carries much more than its share of the estimated cost
        costs = S.tile_costs(w.ctx, w.new, w.q_tile, w.n_q_heads, w.topk, w.block, w.window, w.n_sparse)
        loads = [sum(costs[s.tile0:s.tile0 + s.n_tiles]) for s in shards]
        biggest_tile = max(costs)
        assert max(loads) <= sum(costs) / world + biggest_tile + 1e-6


def test_token_shards_cover_the_rows():
    for total in [1, 7, 64, 1000]:
        for world in [1, 2, 3, 8]:
            rows = []
            for r in range(world):
                lo, hi = S.token_shard(total, r, world)
                rows.extend(range(lo, hi))
            assert rows == list(range(total))


@pytest.mark.parametrize("world", [2, 3])
def test_rank_subproblems_reproduce_the_whole_block(world):
    # ragged chunked MQA prefill, token level with a forced window, two sparse layers
    w = W.Workload("shard", ctx=(0, 70, 5), new=(90, 45, 60), n_q_heads=4, n_kv_heads=1, head_dim=8, q_tile=16,
                   block=1, topk=12, window=6, n_sparse=2)
    rng = np.random.default_rng(5)
    q = rng.standard_normal((w.total_q, 4, 8))
    k = rng.standard_normal((w.total_kv, 1, 8))
    v = rng.standard_normal((w.total_kv, 1, 8))
    layers = [{"q": rng.standard_normal((w.total_q, 4, 8))} for _ in range(w.n_sparse)]
    whole = run_block(q, k, v, layers, w.cu_q(), w.cu_kv(), 1, w.q_tile, w.block, w.topk, w.window)
    shards = _plan(w, world)
    assert shards[0].kind == "q_tiles"
    for s in shards:
        if s.n_tiles == 0:
            continue
        ws = W.scaled(w, ctx=s.ctx, new=s.new)
        nq = ws.total_q
        qs = q[s.q_row0:s.q_row0 + nq]
        ks = k[s.kv_row0:s.kv_row0 + s.kv_rows]
        vs = v[s.kv_row0:s.kv_row0 + s.kv_rows]
        assert ks.shape[0] == ws.total_kv
        ls = [{"q": L["q"][s.q_row0:s.q_row0 + nq]} for L in layers]
        part = run_block(qs, ks, vs, ls, ws.cu_q(), ws.cu_kv(), 1, w.q_tile, w.block, w.topk, w.window)
        rows = tile_rows(w.cu_q(), w.cu_kv(), w.q_tile, range(s.tile0, s.tile0 + s.n_tiles))
        assert rows == list(range(s.q_row0, s.q_row0 + nq))
        assert np.allclose(part["o_full"], whole["o_full"][rows], atol=1e-12, rtol=0)
        assert np.allclose(part["lse_full"], whole["lse_full"][:, rows], atol=1e-12, rtol=0)
        nb = part["scores"].shape[2]
        sc_w = whole["scores"][s.tile0:s.tile0 + s.n_tiles]
        assert np.allclose(part["scores"], sc_w[:, :, :nb], atol=1e-14, rtol=1e-12)
        assert not sc_w[:, :, nb:].any()  # the rank holds every candidate of its tiles
        assert np.array_equal(part["idx"], whole["idx"][s.tile0:s.tile0 + s.n_tiles])
        for a, b in zip(part["layers"], whole["layers"]):
            assert np.allclose(a["o"], b["o"][rows], atol=1e-12, rtol=0)


def _free_port() -> int:
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _gather_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from hybrid_sparse_attention_tma_b200 import shard as SS
        total = 37
        g = torch.Generator().manual_seed(3)
        full = torch.randn((total, 2, 8), generator=g)  # every rank draws the same block
        lo, hi = SS.token_shard(total, rank, world)
        got = SS.all_gather_kv(full[lo:hi].clone(), total)
        q.put((rank, bool(torch.equal(got, full))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_all_gather_the_kv_shards():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            rank, ok = q.get(timeout=240)
            got[rank] = ok
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert got == {0: True, 1: True}
