"""Multi-process host logic of the benchmark with world_size 2 on the gloo
backend (CPU): timings reduce to the max over ranks, and the CPU reference
arm runs and prints on rank 0 only.  Heads are independent, so the GPU path
runs replicas with no data-path collective; only the timing reduction crosses
ranks."""
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


def _worker(rank, world, port, q):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0])
        buf = io.StringIO()
        if rank != 0:
            class Args:
                steps, warmup = 1, 0
            with redirect_stdout(buf):
                bench.reference_arm(Args())
        q.put((rank, got, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_rank0_only_reference():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, printed in out:
        assert got == [2.0, 10.0, 5.0]
        if rank != 0:
            assert printed == ""
