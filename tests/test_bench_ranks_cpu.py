"""The benchmark's multi-rank logic on CPU: world_size-2 gloo ranks (127.0.0.1).

The layer runs as independent replicas (no data-path collective); the only
cross-rank steps are the barrier and the max over ranks of the measured step
time, from which the whole-job throughput is computed.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        # rank r measured (r + 1) * 1.5 ms per step; the job's step time is the slowest rank's
        t = bench.max_over_ranks((rank + 1) * 1.5, dist, "cpu")
        q.put((rank, t, bench.aggregate_tokens_per_s(4096, world, t)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, tps in res:
        assert t == pytest.approx(3.0)
        assert tps == pytest.approx(4096 * 2 / 3.0e-3)


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5) == 2.5
    assert bench.aggregate_tokens_per_s(4096, 1, 0.5) == pytest.approx(8192000.0)
