"""Multi-process host logic of the replicas-only multi-GPU mode, on CPU with gloo.

The path shards by sequence with no exchange step: every rank runs an independent replica of
the workload and the only collective is the max-reduction of the timing. These tests run two
gloo ranks on the CPU and check that reduction, the aggregate throughput, and that the seeded
inputs each replica draws are identical.
"""
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


def _worker(rank, world, port, results):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import workloads
    barrier, max_over_ranks = bench.dist_helpers(world, torch.device("cpu"))
    barrier()
    local_ms = 10.0 + 5.0 * rank
    ms = max_over_ranks(local_ms)
    value = bench.aggregate_throughput(world, 8, 20, ms)
    wi = workloads.generate(workloads.WORKLOADS["tiny"])
    digest = float(wi.layers[0].q.float().sum()) + float(wi.layers[0].k_cache.float().sum())
    barrier()
    dist.destroy_process_group()
    results[rank] = (ms, value, digest)


def test_two_rank_replicas():
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    ms0, v0, d0 = results[0]
    ms1, v1, d1 = results[1]
    assert ms0 == ms1 == 15.0
    assert v0 == v1 == pytest.approx(2 * 8 * 20 / 0.015)
    assert d0 == d1
