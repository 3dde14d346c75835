"""The N > 1 host path of bench.py on CPU ranks (gloo, world size 2): each
rank times its own copy of the workload, the job time is the max over ranks
and the whole-job value counts every rank's bytes."""
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


def _rank(rank, world, port, q):
    import datetime
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank          # rank 1 is the slow one
        job = bench.max_over_ranks(mine, dist, "cpu")
        dist.barrier()
        q.put((rank, job, bench.weak_scaling_gbs(1000, 4, world, job)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]
    # 1000 bytes x 4 steps x 2 ranks in 15 ms
    assert abs(res[0][2] - 1000 * 4 * 2 / 0.015 / 1e9) < 1e-12


def test_single_process_path():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.weak_scaling_gbs(268697600, 10, 1, 0.5) == pytest.approx(268697600 * 10 / 5e-4 / 1e9)
