"""Multi-process host logic of bench.py on CPU (gloo, world size 2): every
rank runs its own replica, timings take the slowest rank and the value is the
whole job's units over that time; the reference arm prints on rank 0 only."""
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
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    units = 100.0 * (rank + 1)          # rank r processed 100 (r + 1) units
    ms = 2.0 + rank                     # in 2 + r milliseconds
    rate, slowest = bench.whole_job_rate(units, ms, dist, device="cpu")
    out[rank] = (rate, slowest, bench.max_over_ranks(float(rank), dist, "cpu"),
                 bench.sum_over_ranks(1.0, dist, "cpu"))
    dist.barrier()
    dist.destroy_process_group()


def test_whole_job_rate_over_two_gloo_ranks():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a threaded process
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    for rank in (0, 1):
        rate, slowest, mx, sm = res[rank]
        assert slowest == 3.0                       # the slower rank's time
        assert rate == pytest.approx(300.0 / 3e-3)  # all units / slowest time
        assert mx == 1.0 and sm == 2.0


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode == 0 and r.stdout.strip() == ""
