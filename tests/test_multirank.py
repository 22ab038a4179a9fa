"""The multi-rank path of bench.py on CPU (gloo, world size 2): ranks are independent replicas,
timings are combined as the maximum over ranks, and only rank 0 prints the JSON line."""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank: int, world: int, port: int, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank), "DELTA_DIST_BACKEND": "gloo"})
    sys.path.insert(0, ROOT)
    import torch
    import bench
    dist, r, w, _ = bench.dist_init()
    try:
        dev = torch.device("cpu")
        bench.barrier(dist, dev)
        out[rank] = bench.max_over_ranks(dist, 10.0 * (rank + 1), dev)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_is_the_slowest_rank():
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_max_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 20.0, 1: 20.0}


def test_two_rank_reference_arm_prints_once():
    port = _free_port()
    env = dict(os.environ, DELTA_DIST_BACKEND="gloo")
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
                        "--impl", "reference", "--config", "1", "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
