"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, each with its own time, agree on
the slowest rank's time and on the total number of query tokens (the path itself has no
collective: every rank runs an independent replica)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    ws, r = bench.init_dist("gloo")
    bench.barrier(ws)
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, ws, torch.device("cpu"))
    tokens = bench.sum_over_ranks(32 * (rank + 1), ws, torch.device("cpu"))
    bench.barrier(ws)
    q.put((r, ws, slowest, tokens))
    dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_time_and_total_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 2, 15.0, 96.0), (1, 2, 15.0, 96.0)]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.sum_over_ranks(7, 1, None) == 7.0
