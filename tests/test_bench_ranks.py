"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): every rank
sees the max of the per-rank times, the job rate counts all replicas, and
`bench.py --gpus 2` started as a plain process relaunches itself with one
rank per replica and reports n_gpus = 2."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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


def test_gpus_flag_launches_one_rank_per_replica():
    env = dict(os.environ, PYTHONPATH=ROOT)
    env.pop("WORLD_SIZE", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--steps", "3",
                        "--warmup", "3", "--rank-selftest"], capture_output=True, text=True, timeout=240, env=env,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout                  # rank 0 alone prints
    j = json.loads(lines[0])
    assert j["n_gpus"] == 2
    # the slow replica (rank 1: 20 ms per step) sets the job time
    assert j["ms_per_step"] == pytest.approx(20.0)
    assert j["value"] == pytest.approx(100.0 * 2 * 3 / 0.060)


def test_world_size_must_match_gpus():
    env = dict(os.environ, PYTHONPATH=ROOT, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--rank-selftest"],
                       capture_output=True, text=True, timeout=120, env=env, cwd=ROOT)
    assert r.returncode == 2
    assert "WORLD_SIZE=1" in r.stdout
