"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): the
max-over-ranks timing reduction and the whole-job throughput aggregation.
No GPU and no data-path collective are involved: the operator shards over
independent (batch, head) problems, so ranks only agree on the timing."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench.dist_env()
        assert (r, lr, w) == (rank, rank, world)
        bench.barrier()
        m = bench.max_over_ranks(times[rank])
        value, ms = bench.aggregate(w, 1e12, 10, m)
        q.put((rank, m, value, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_gloo():
    world = 2
    times = [0.5, 0.8]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, m, value, ms in res:
        assert m == pytest.approx(0.8)              # every rank sees the slowest rank's time
        assert value == pytest.approx(2 * 10 / 0.8)  # all ranks' FLOPs / slowest time, TFLOP/s
        assert ms == pytest.approx(80.0)


def test_single_process_identity():
    assert bench.max_over_ranks(1.25) == 1.25
    value, ms = bench.aggregate(1, 2e12, 4, 2.0)
    assert value == pytest.approx(4.0) and ms == pytest.approx(500.0)
