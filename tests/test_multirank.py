"""Host logic of the N-rank bench on CPU: two gloo ranks share one block.

Each rank draws the whole block from the same seed and keeps its shard
(hybrid_sparse_attention_tma_b200.shard): for an MQA prefill that is a range
of selection tiles whose K / V arrive by all-gather of the ranks' token
shards. The ranks' new tokens add up to the block's; the gathered K / V slice
equals the block's rows; timings are combined as the max over ranks, outside
the timed region; the job's rate is the block's tokens over the slowest rank.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as W
        from hybrid_sparse_attention_tma_b200 import shard as S
        w = W.Workload("mr", ctx=(0, 40), new=(96, 64), n_q_heads=4, n_kv_heads=1, head_dim=64, q_tile=16,
                       block=1, topk=24, window=8, n_sparse=1)
        w_r, inp, kv_own = bench.rank_problem(w, world, rank, "cpu")
        full = W.make_block_inputs(w, device="cpu", seed=bench.block_seed(w))
        k_own, v_own, total, r0, n = kv_own
        kf = S.all_gather_kv(k_own, total)
        kv_ok = bool(torch.equal(kf, full.k)) and bool(torch.equal(kf[r0:r0 + n], inp.k))
        q_ok = bool(torch.equal(inp.q, full.q[S.plan(w.ctx, w.new, 4, 1, 16, world, 24, 1, 8, 1)[rank].q_row0:][
            :w_r.total_q]))
        # per-rank timings: rank r is slower on the first entry, faster on the second
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 1.5], "cpu")
        rate = bench.whole_job_rate(w.total_q, mx[0])
        q.put((rank, w_r.total_q, kv_ok, q_ok, mx, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_one_block():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            rank, toks, kv_ok, q_ok, mx, rate = q.get(timeout=240)
            got[rank] = (toks, kv_ok, q_ok, mx, rate)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert sorted(got) == [0, 1]
    assert got[0][0] + got[1][0] == 160 and got[0][0] > 0 and got[1][0] > 0  # the block's tokens, split
    assert all(got[r][1] and got[r][2] for r in range(world))
    for r in range(world):
        assert got[r][3] == [11.0, 5.0, 1.5]
    assert got[0][4] == pytest.approx(160 / (11.0 / 1e3))
    assert got[0][4] == got[1][4]


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not (dist.is_available() and dist.is_initialized())
    assert bench.max_over_ranks([3.0, 1.0], "cpu") == [3.0, 1.0]
    assert bench.whole_job_rate(1000, 2.0) == pytest.approx(500000.0)
