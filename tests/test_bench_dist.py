"""The multi-process plumbing of bench.py on host-only ranks (gloo, world size 2): the
rendezvous, the barrier, the max-over-ranks device time, the whole-job throughput of
independent replicas, and the reference arm running on rank 0 only."""
import contextlib
import io
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


def _worker(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2",
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    class A:
        gpus, steps, warmup = 2, 3, 3
    ws, r, local = bench.dist_setup(A)
    try:
        assert (ws, r, local) == (2, rank, rank) and dist.get_backend() == "gloo"
        bench.barrier(ws)
        slow = bench.max_over_ranks(ws, 10.0 + 5.0 * rank)   # rank 1 is the slower one
        thr = bench.replica_throughput(ws, 512, 4, slow)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            if rank != 0:
                bench.run_reference(A, ws, r, "tiny")   # other ranks exit without work
        q.put((rank, slow, thr, buf.getvalue()))
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_two_host_ranks_max_time_and_replica_throughput():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    mp.start_processes(_worker, args=(_free_port(), q), nprocs=2, join=True, start_method="spawn")
    got = sorted(q.get() for _ in range(2))
    for rank, slow, thr, out in got:
        assert slow == 15.0                       # the slowest rank's time, seen by both ranks
        assert thr == pytest.approx(2 * 512 * 4 / 0.015)
    assert got[1][3] == ""                        # rank 1 printed nothing for the reference arm
