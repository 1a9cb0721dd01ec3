"""The multi-rank plumbing of bench.py with two gloo ranks on CPU: replicas
of the workload (weak scaling, no data-path collective), a barrier, and the
max over ranks of the per-rank device time."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    w, r, lr = bench.dist_setup()
    assert (w, r, lr) == (world, rank, rank)
    bench.barrier(w)
    ms_local = 10.0 + 5.0 * rank            # the slower rank decides
    ms = bench.max_over_ranks(ms_local, w)
    value = bench.aggregate_throughput(4096, ms, w)
    out[rank] = (ms, value)
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_report_the_slowest_rank():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1]
    ms, value = out[0]
    assert ms == 15.0
    assert value == pytest.approx(4096 * 2 / 0.015)


def test_single_rank_aggregate_is_plain_throughput():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.aggregate_throughput(4096, 2.0, 1) == pytest.approx(2048000.0)
