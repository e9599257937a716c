"""The multi-GPU plumbing of bench.py on two CPU ranks (gloo): process-group setup from the
torchrun environment, the max-over-ranks timing, barriers, the whole-job throughput of the
weak-scaling layout (every rank scans its own batch; no data-path collective), and the
reference arm running on rank 0 only."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    try:
        w, r, local = bench.dist_setup(world, backend="gloo")
        assert (w, r, local) == (world, rank, rank)
        bench.barrier(w)
        t = bench.max_over_ranks(1.0 + rank, w)          # rank r "took" 1 + r seconds
        v = bench.job_throughput(1000, w, 4, t)
        # reference arm: only rank 0 works and prints; the others return at once
        buf = io.StringIO()
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(None, w, rank)
        bench.barrier(w)
        q.put((rank, t, v, buf.getvalue()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, v, out in res:
        assert t == pytest.approx(2.0)                   # the slowest rank's time, on every rank
        assert v == pytest.approx(1000 * 2 * 4 / 2.0 / 1e9)
        if rank != 0:
            assert out == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        assert bench.dist_setup(1) == (1, 0, 0)
        assert bench.max_over_ranks(3.5, 1) == 3.5
        assert bench.job_throughput(41943040, 1, 10, 3.0e-3) == pytest.approx(139.81, rel=1e-3)
    finally:
        os.environ.update(env)
