"""The multi-GPU path of the benchmark is replicas only: each rank runs the
whole hot path on its own GPU and the ranks exchange nothing but a barrier
and two scalars.  This checks that plumbing with two gloo ranks on the CPU:
the max over ranks of the step time, the sum of bytes, and the resulting
whole-job throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench

    d = bench.Dist(backend="gloo")
    d.init()
    try:
        d.barrier()
        # rank r moved (r + 1) GB in (10 + r) ms per step
        gbs, ms = bench.aggregate_throughput((rank + 1) * 1e9, 10.0 + rank, d)
        q.put((rank, gbs, ms, d.max(float(rank)), d.sum(1.0)))
    finally:
        d.close()


@pytest.mark.parametrize("world", [2])
def test_replica_aggregation_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, gbs, ms, mx, sm in results:
        assert ms == 10.0 + (world - 1)            # the slowest rank's time
        assert mx == float(world - 1)
        assert sm == float(world)
        total = sum(r + 1 for r in range(world)) * 1e9
        assert abs(gbs - total / (ms * 1e-3) / 1e9) < 1e-9


def test_single_process_needs_no_process_group():
    import bench

    d = bench.Dist(backend="gloo")
    d.init()
    assert d.pg is None and d.max(3.0) == 3.0 and d.sum(2.0) == 2.0
    gbs, ms = bench.aggregate_throughput(2e9, 4.0, d)
    assert ms == 4.0 and abs(gbs - 500.0) < 1e-9
