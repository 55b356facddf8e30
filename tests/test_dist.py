"""The replicas path of bench.py on more than one rank, on the host: two
processes with the gloo backend (no GPU). Replicas exchange nothing on the data
path; the only collectives are the barrier and the max of the timed region."""
import json
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
    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup(argparse.Namespace(impl="reference"))
    assert (r, w, local) == (rank, world, rank)
    bench.dist_barrier(w)
    m = bench.dist_max(float(10 * (rank + 1)), w)
    out[rank] = m
    dist.destroy_process_group()


def test_dist_helpers_two_ranks_gloo():
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert dict(out) == {0: 20.0, 1: 20.0}


def test_reference_arm_under_torchrun_two_ranks():
    """`bench.py --impl reference --gpus 2` launched like the driver launches it:
    rank 0 alone runs the oracle and prints one JSON line, every rank exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "3"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
