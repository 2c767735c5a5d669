"""The multi-GPU host logic of bench.py on two gloo ranks (CPU only).

With N > 1 each rank runs its own micro-batch (weak scaling, no collective in the data
path); the only cross-rank steps are the barriers around the timed region and the max
over ranks of the elapsed time. This runs those helpers on a world of two CPU processes.
"""

import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

from tests.conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench._dist_setup(world)
    assert (r, w, local) == (rank, world, rank)
    assert dist.get_backend() == "gloo"
    bench._barrier_sync(w)
    elapsed = 10.0 * (rank + 1)          # each rank reports its own step time
    worst = bench._max_over_ranks(elapsed, w)
    bench._barrier_sync(w)
    dist.destroy_process_group()
    q.put((rank, worst))


@pytest.mark.skipif(torch.cuda.is_available(), reason="exercises the gloo (CPU) path")
def test_two_rank_barrier_and_max_over_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    results = dict(q.get(timeout=5) for _ in range(world))
    assert results == {0: 20.0, 1: 20.0}
