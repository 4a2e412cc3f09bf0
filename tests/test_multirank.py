"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The estimators partition by environment rows, so ranks run independent
shards with no data-path collective; the only cross-rank steps are the
barrier and the max over ranks of the device-timed duration.  These run
here as two gloo processes.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        elapsed = [12.5, 20.0][rank]
        mx = bench.max_over_ranks(elapsed)
        calls = bench.workload_calls("gae_64x32", rank)
        shape = calls[0][2]["rewards"].shape
        first = float(calls[0][2]["rewards"][0, 0])
        dist.barrier()
        q.put((rank, mx, shape, first))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_shards():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(2))
    # both ranks see the slowest rank's time
    assert res[0][1] == res[1][1] == 20.0
    # same shard shapes, different data
    assert res[0][2] == res[1][2] == (64, 32)
    assert res[0][3] != res[1][3]


def test_aggregate_rate_and_single_rank_max():
    import bench
    assert bench.aggregate_rate(4, 1000, 2.0) == pytest.approx(2.0e6)
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.shard_seed(1000, 0) == 1000 and bench.shard_seed(1000, 2) != 1000
