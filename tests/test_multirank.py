"""The N > 1 path of bench.py on CPU: world-size-2 gloo ranks agree on the
slowest rank's time and the whole-job throughput aggregates all ranks. (The
workloads run one independent replica per GPU; this is the only exchange.)"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 50.0 * rank  # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, "cpu")
        out[rank] = (ms, bench.job_throughput(1e12, world, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 150.0
    assert out[0][1] == pytest.approx(2e12 / 0.150)


def test_single_rank_passthrough():
    import bench
    assert bench.max_over_ranks(12.5) == 12.5
    assert bench.job_throughput(3.0, 1, 1000.0) == 3.0
