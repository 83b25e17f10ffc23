"""The benchmark's multi-rank host logic on CPU with gloo, world size 2: independent per-rank
problems (weak scaling, no data-path collective), job time = max over ranks, kernel counts summed,
and only rank 0 runs and prints the reference arm."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    t, n = bench.aggregate(10.0 * (rank + 1), 7 * (rank + 1), world, torch.device("cpu"))
    out.put((rank, t, n, bench.rank_seed(5, rank)))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_max_time_and_summed_launches_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [20.0, 20.0]          # max over ranks, seen by every rank
    assert [r[2] for r in res] == [21, 21]              # launches summed
    assert res[0][3] != res[1][3]                       # independent problems per rank


def test_reference_arm_only_rank0_runs():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True,
                       text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
