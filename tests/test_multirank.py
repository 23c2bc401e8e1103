"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own
replica. The reported time is the maximum over ranks and the throughput is
all ranks' units over that time (no data-path collective exists)."""

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


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench

    d = bench.Dist()
    assert d.backend == "gloo"
    d.barrier()
    local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
    ms = d.max(local_ms)
    thr = bench.replica_throughput(1e12, ms, d.world)
    out[rank] = (ms, thr)
    d.close()


def test_two_gloo_ranks_max_and_aggregate():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()  # no fork of this (possibly threaded) process
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        ms, thr = out[r]
        assert ms == 15.0                  # max over ranks
        assert thr == pytest.approx(2 * 1e12 / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        d = bench.Dist()
        assert d.pg is None and d.max(3.0) == 3.0
    finally:
        os.environ.update(env)
