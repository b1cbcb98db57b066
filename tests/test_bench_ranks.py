"""The bench's multi-rank bookkeeping on CPU (gloo, world size 2).

The path needs no exchange, so `bench.py --gpus N` runs N independent
replicas: the job's time is the slowest rank's (a MAX all-reduce), and the
reference arm is printed by rank 0 alone while the other ranks exit 0
without work.  Both are host logic and run here without a GPU.
"""
import datetime
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, values, queue):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        sys.path.insert(0, ROOT)
        import bench

        queue.put((rank, bench.max_over_ranks(values[rank], dist, "cpu")))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    values = [0.25, 1.75]
    port = _free_port()
    procs = [ctx.Process(target=_max_worker, args=(r, 2, port, values, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0]
    got = dict(queue.get(timeout=10) for _ in range(2))
    assert got == {0: 1.75, 1: 1.75}


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5


def test_reference_arm_two_ranks():
    """torchrun with 2 ranks: one JSON line from rank 0, exit 0 everywhere."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "0", "--cpu-rows", "4"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    out = json.loads(lines[0])
    assert out["impl"] == "reference"
    assert out["n_gpus"] == 2
    assert out["value"] > 0 and out["unit"] == "GB/s"
    assert out["e2e"] == {"value": out["value"], "unit": "GB/s",
                          "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert out["cpu_baseline"]["kind"] == "oracle"
