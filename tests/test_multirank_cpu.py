"""The N > 1 path of bench.py on CPU: world_size-2 gloo ranks.

The layer does not shard in this build (replicas only), so the multi-rank
logic is the timing reduction: every rank times the same K steps, the job's
time is the slowest rank's, and the value counts every rank's tokens.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import sys
        sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
        import bench
        mine = [12.5, 40.0][rank]
        slowest = bench.max_over_ranks(mine, world)
        value = bench.replica_throughput(8192, world, 10, slowest)
        second = bench.max_over_ranks(-float(rank), world)  # a second call in the same order
        q.put((rank, slowest, value, second))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_value_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value, second in got:
        assert slowest == 40.0
        assert value == pytest.approx(2 * 8192 * 10 / 0.040)
        assert second == 0.0


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_throughput(64, 1, 2, 1000.0) == pytest.approx(128.0)
