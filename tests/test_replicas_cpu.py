"""Multi-GPU path of bench.py on CPU: replicas only (one independent request
per rank, no data-path collective); torch.distributed carries the barrier and
the max over ranks of the timed region.  world_size 2, gloo, 127.0.0.1."""
import os
import socket

import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), BENCH_BACKEND="gloo")
    import bench
    r, local, ws = bench._dist()
    bench._barrier(ws)
    # each replica times its own work; the job time is the slowest rank
    t = bench._max_over_ranks(10.0 * (rank + 1), ws, torch.device("cpu"))
    q.put((r, local, ws, t))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_replicas_take_max_over_ranks_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out == [(0, 0, 2, 20.0), (1, 1, 2, 20.0)]
