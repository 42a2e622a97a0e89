"""Multi-rank aggregation of bench.py on CPU (gloo, world size 2): every rank
sees the max of the per-rank times, and the job rate counts all replicas."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    local_ms = 10.0 * (rank + 1)                       # rank 1 is the slow replica
    mx = bench.reduce_max_ms(local_ms, world)
    rate = bench.job_rate(100.0, world, 5, mx)
    dist.barrier()
    out[rank] = (mx, rate)
    dist.destroy_process_group()


def test_reduce_max_and_job_rate_two_ranks():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 20.0
    # 100 units per rank-step, 2 ranks, 5 steps, in 20 ms
    assert res[0][1] == pytest.approx(100.0 * 2 * 5 / 0.020)


def test_single_rank_identity():
    import bench
    assert bench.reduce_max_ms(3.5, 1) == 3.5
    assert bench.job_rate(10, 1, 2, 4.0) == pytest.approx(5000.0)
