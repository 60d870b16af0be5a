"""The multi-process path of bench.py on CPU: two gloo ranks, one process each.

Every rank runs its own replica of the workload (independent batch rows, no
collective on the data path); the only collectives are the timing barrier and
the max over ranks of the device time. Here each rank reports a different
time and a different replica seed; the max must be the largest rank's value
and the replicas' inputs must differ.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import numpy as np
    import torch.distributed as dist

    import bench
    import e2ttt_inputs as gen
    r, w, lr_ = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    dist.barrier()
    t = bench.max_over_ranks(10.0 + 5.0 * r, w)
    wl = gen.BY_NAME["tiny_linear"]
    x = gen.generate(wl, seed=wl.seed + 1000 * r)
    digest = float(np.sum(x["q"][0, 0, :4]))
    dist.destroy_process_group()
    q.put((r, w, lr_, t, digest))


@pytest.mark.parametrize("world", [2])
def test_two_rank_timing_reduction(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[0] for r in res] == list(range(world))
    assert all(r[1] == world and r[2] == r[0] for r in res)
    assert all(r[3] == 10.0 + 5.0 * (world - 1) for r in res)  # max over ranks
    assert res[0][4] != res[1][4]                               # distinct replicas


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
