"""Multi-rank host logic of bench.py on CPU: world_size 2 over gloo.

bench.py runs independent replicas (one per GPU); the only collectives are the
timing barrier and the max over ranks of the device time. These tests run that
logic with two gloo processes, and check that the reference arm under a
multi-rank launch prints from rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 20.0][rank]
        m = bench.max_over_ranks(local_ms, dist, "cpu")
        dist.barrier()
        q.put((rank, m, bench.job_gbs(world, 1_000_000, 10, m)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert [g[1] for g in got] == [20.0, 20.0]
    # 2 ranks x 1e6 bytes x 10 steps in 20 ms
    assert got[0][2] == pytest.approx(2 * 1e6 * 10 / 0.020 / 1e9)


def test_single_process_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.job_gbs(1, 2e9, 1, 1000.0) == pytest.approx(2.0)


def test_reference_arm_prints_on_rank0_only():
    env = dict(os.environ)
    out = {}
    for rank in (0, 1):
        env.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                            "--warmup", "3", "--ref-seconds", "0.5"], capture_output=True, text=True, env=env,
                           timeout=300)
        assert r.returncode == 0, r.stderr
        out[rank] = r.stdout.strip()
    assert out[1] == ""
    line = json.loads(out[0].splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
