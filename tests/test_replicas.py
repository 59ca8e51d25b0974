"""Host-side logic of the multi-GPU bench (replicas only), with gloo ranks on CPU.

bench.py runs one independent replica per GPU; the only cross-rank steps are
the barrier and the reduction of the timing scalars: whole-job units summed
over ranks, time = the slowest rank's."""

import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        units = 100.0 * (rank + 1)           # rank r processed 100 (r+1) units
        secs = 0.5 + rank                    # and took 0.5 + r seconds
        total, tmax = bench.aggregate(units, secs, dist)
        dist.barrier()
        q.put((rank, total, tmax))
    finally:
        dist.destroy_process_group()


def test_aggregate_sums_units_and_takes_max_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, total, tmax in out:
        assert total == 300.0
        assert tmax == 1.5


def test_aggregate_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.aggregate(7.0, 2.0, None) == (7.0, 2.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_bench_rejects_too_few_warmup_steps():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode != 0
