"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The codec path partitions into independent segments, so ranks never exchange data: each rank codes
its own seeded workload (weak scaling) and the only collective is the max over ranks of the elapsed
time. This test runs that plumbing with two gloo ranks and the CPU oracle standing in for the GPU
work: per-rank inputs differ, every rank's stream round-trips, and the reported value uses the
slowest rank's time.
"""
import os
import socket

import numpy as np
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        from entropy_coded_lossless_b200 import inputs

        x = inputs.laplace_int8(20_000, 7.258, seed=100 + rank).numpy()  # the rank's own data
        stream, _ = oracle.encode(x, 16, 7, 4, 4096)
        rc, y = oracle.decode(stream)
        ok = rc == 0 and np.array_equal(y, x.view(np.uint8))
        ms = 10.0 + rank  # a stand-in per-rank elapsed time
        ms_max = bench.max_over_ranks(ms, "cpu")
        digest = torch.tensor([int(x.view(np.uint8).astype(np.int64).sum())], dtype=torch.int64)
        gathered = [torch.zeros_like(digest) for _ in range(world)]
        dist.all_gather(gathered, digest)
        results[rank] = (ok, ms_max, bench.whole_job_gbs(x.size, world, ms_max), [int(g) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")  # no fork: the test process may already run threads
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert len(results) == world
    for r in range(world):
        ok, ms_max, value, digests = results[r]
        assert ok
        assert ms_max == pytest.approx(11.0)
        assert value == pytest.approx(2 * 20_000 / 11e-3 / 1e9)
        assert digests[0] != digests[1]  # each rank coded its own data
