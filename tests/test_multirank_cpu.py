"""The multi-rank plumbing of bench.py (weak scaling: barriers, the max of
the per-rank times, the sum of the per-rank work) with two gloo ranks on the
CPU; the GPU run uses the same calls over NCCL."""
import os
import socket
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        t_max = bench.max_over_ranks(1.5 + rank, world)   # per-rank times 1.5 and 2.5
        f_sum = bench.sum_over_ranks(10.0 * (rank + 1), world)  # per-rank work 10 and 20
        bench.barrier(world)
        q.put((rank, t_max, f_sum))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_summed_work():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t_max, f_sum in res:
        assert t_max == 2.5  # the job time is the slowest rank's
        assert f_sum == 30.0  # whole-job work adds over ranks
