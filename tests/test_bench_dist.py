"""The bench's multi-rank plumbing on CPU: two gloo ranks set up the group
the way torchrun launches them, meet at the barrier, agree on the slowest
rank's time and compute the whole-job rate from it."""
import os
import socket
import sys
import time

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(ws), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(ws, backend="gloo")
    assert (w, r) == (ws, rank)
    bench.barrier(w)
    ms = 10.0 + 5.0 * rank                       # the slower rank decides
    m = bench.max_over_ranks(ms, w)
    out[rank] = (m, bench.whole_job_rate(1000, w, m))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    ws = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.spawn(_rank, args=(ws, _free_port(), out), nprocs=ws, join=False)
    deadline = time.time() + 180
    while not ctx.join(timeout=5):          # True once every rank has exited
        assert time.time() < deadline, "ranks did not finish"
    for r in range(ws):
        m, rate = out[r]
        assert m == 15.0
        assert rate == pytest.approx(ws * 1000 / 0.015)


def test_single_rank_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.whole_job_rate(10, 1, 1000.0) == pytest.approx(10.0)
