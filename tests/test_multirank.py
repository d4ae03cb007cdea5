"""Host logic of the N-rank bench on CPU: two gloo ranks.

Every rank processes its own independent hybrid block (distinct seed, hence
distinct inputs); the only collective is the max over ranks of the timings,
taken outside the timed region; the whole-job rate is every rank's tokens over
the slowest rank's step time.
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
        w = W.WORKLOADS["tiny"]
        seed = bench.rank_seed(w, rank)
        inp = W.make_block_inputs(w, device="cpu", seed=seed)
        digest = float(inp.q.float().abs().sum()) + float(inp.k.float().abs().sum())
        # per-rank timings: rank r is slower on the first entry, faster on the second
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 1.5], "cpu")
        rate = bench.whole_job_rate(world, w.total_q, mx[0])
        q.put((rank, seed, digest, mx, rate))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_blocks_and_max_timing():
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
            rank, seed, digest, mx, rate = q.get(timeout=240)
            got[rank] = (seed, digest, mx, rate)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert sorted(got) == [0, 1]
    # independent blocks: distinct seeds and inputs
    assert got[0][0] != got[1][0]
    assert got[0][1] != pytest.approx(got[1][1])
    # every rank sees the element-wise max over ranks
    for r in range(world):
        assert got[r][2] == [11.0, 5.0, 1.5]
    # whole-job rate: both ranks' tokens over the slowest rank's time
    import workloads as W
    tokens = W.WORKLOADS["tiny"].total_q
    assert got[0][3] == pytest.approx(world * tokens / (11.0 / 1e3))
    assert got[0][3] == got[1][3]


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not (dist.is_available() and dist.is_initialized())
    assert bench.max_over_ranks([3.0, 1.0], "cpu") == [3.0, 1.0]
    assert bench.whole_job_rate(1, 1000, 2.0) == pytest.approx(500000.0)
