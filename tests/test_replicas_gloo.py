"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own replica.

The decode step does not shard without an exchange per layer, so N GPUs run N
independent replicas and the job's throughput is every rank's tokens over the slowest
rank's time.  This checks that aggregation, the barrier, and that only rank 0 of the
reference arm does work.
"""
import os
import socket
import sys

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # rank r took (r + 1) * 100 ms for 10 steps of a batch of 8
        ms, value = bench.job_throughput(world, (rank + 1) * 100.0, 10, 8)

        class A:
            workload, warmup, steps, gpus = "tiny-b1", 0, 1, world

        ref = bench.run_reference(A, world, rank) if rank != 0 else None
        bench.barrier(world)
        out.put((rank, ms, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value, ref in res:
        assert abs(ms - 20.0) < 1e-9           # the slowest rank: 200 ms / 10 steps
        assert abs(value - 2 * 8 / 0.020) < 1e-6  # both ranks' tokens over that time
        assert ref is None                      # rank 1 of the reference arm does nothing
