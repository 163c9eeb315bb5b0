"""The multi-GPU path of bench.py on CPU: two gloo ranks (replicas only; the
path has no data-path collective).  Checks the max-over-ranks timing, the
whole-job rate and that only rank 0 runs the reference arm."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r "took" 10 * (r + 1) ms: every rank sees the slowest rank's time
        m = bench.max_over_ranks(10.0 * (rank + 1), "cpu")
        rate = bench.whole_job_rate(world, 100, m)

        class A:
            steps, gpus = 1, world
        buf = io.StringIO()
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(A(), rank)  # returns at once on ranks other than 0
        dist.barrier()
        out[rank] = (m, rate, buf.getvalue())
    finally:
        dist.destroy_process_group()


def test_two_replicas_max_over_ranks_and_rate():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as mgr:  # (no fork of a threaded process)
        out = mgr.dict()
        mp.start_processes(_rank, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0
    assert res[0][1] == res[1][1] == world * 100 / 0.020  # 10,000 items/s for the whole job
    assert res[1][2] == ""  # rank 1 printed nothing for the reference arm


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.whole_job_rate(1, 10, 1000.0) == 10.0
