"""The multi-process path of bench.py on CPU: two gloo ranks reduce their
timings to the max over ranks and their units to the job total."""
import os
import socket
import sys
from datetime import timedelta

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench

    env = bench.dist_env()
    t, u = bench.reduce_timing(1.5 + rank, 100 * (rank + 1))
    queue.put((rank, env, t, u))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_timing_reduction():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, env, t, u in results:
        assert env == (2, rank, rank)
        assert t == 2.5          # the slowest rank's time
        assert u == 300          # units of the whole job
    # whole-job throughput as bench.py reports it
    assert results[0][3] / results[0][2] == 120.0


def test_single_process_reduction_is_identity():
    import bench

    assert bench.reduce_timing(0.25, 7) == (0.25, 7)
