"""The multi-process path of bench.py on CPU (gloo, world size 2).

bench.py runs one process per GPU; every rank works on an independent
problem (replicas, no data-path collective) and the job's time is the
maximum over ranks.  These tests run that host logic with the gloo backend:
the rendezvous, the max-over-ranks reduction and the barrier, and the
reference arm under torchrun, where rank 0 alone prints one JSON line.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import torch

    import bench
    r, w, local = bench.dist_setup(None)
    assert (r, w, local) == (rank, world, rank)
    # every rank reports its own device time; the job time is the largest
    got = bench.dist_max(10.0 + 5.0 * rank, w, torch.device("cpu"))
    bench.dist_barrier(w)
    out[rank] = got
    bench.dist_done(w)


def test_two_ranks_take_the_max_of_their_times():
    port = _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import torch

    import bench
    env = {k: os.environ.pop(k) for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK") if k in os.environ}
    try:
        assert bench.dist_setup(None) == (0, 1, 0)
        assert bench.dist_max(3.5, 1, torch.device("cpu")) == 3.5
    finally:
        os.environ.update(env)


@pytest.mark.slow
def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0",
           "--ref-seconds", "2"]
    env = dict(os.environ, OMP_NUM_THREADS="2")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
