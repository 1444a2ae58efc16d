"""The N > 1 path of bench.py is replicas only: each rank runs its own copy of
the workload and the only collectives are a barrier and a max over ranks.
Checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local = [10.0 + rank, 3.0 - rank]          # per-rank step and e2e times (ms)
        got = bench.max_over_ranks(local, torch.device("cpu"), world)
        dist.barrier()
        q.put((rank, got, bench.replica_throughput(1000.0, got[0], world)))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in res:
        assert got == [11.0, 3.0]                  # the slowest rank's time, on every rank
        assert thr == pytest.approx(2 * 1000.0 / 11e-3)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], None, 1) == [1.5, 2.5]
    assert bench.replica_throughput(100.0, 2.0, 1) == pytest.approx(5e4)
