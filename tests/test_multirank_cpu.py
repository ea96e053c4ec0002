"""The benchmark's multi-GPU logic on CPU: world-size-2 gloo process group.

The path has no exchange step (independent replicas), so the only cross-rank
logic is the max-over-ranks timing and the whole-job aggregation; both are
exercised here with ranks that report different times.  Also the per-rank
work split: every rank runs the same workload (weak scaling).
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        my_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        worst = bench.max_over_ranks(my_ms, dist, "cpu")
        rate = bench.aggregate_rate(world, 4.0e12, worst / 1e3, 1e12)
        dist.barrier()
        q.put((rank, worst, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, rate in res:
        assert worst == pytest.approx(15.0)           # the slowest rank's time
        assert rate == pytest.approx(2 * 4.0 / 0.015)  # both replicas' work / max time


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.aggregate_rate(1, 2e12, 0.5, 1e12) == pytest.approx(4.0)
