"""Multi-rank host paths of bench.py on CPU (gloo, world size 2).

The score / resample / remap path shards by sequence with no data-path
collective; what runs across ranks is the timing plumbing (barrier, the max over
ranks of the device time) and the launch contract (one process per rank under
torch.distributed.run, rank 0 alone prints).  These run on the host only.
"""

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


def _worker(rank, world, port, values, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, _ = bench.dist_init()
    try:
        bench.barrier(w)
        out[r] = bench.max_over_ranks(values[r], w)
        bench.barrier(w)
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    values = [3.5, 7.25]
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, values, out), nprocs=world, join=True)
        assert dict(out) == {0: 7.25, 1: 7.25}


def test_reference_arm_under_torchrun_two_ranks():
    """bench.py --impl reference launched as the driver does for N = 2: rank 0
    prints exactly one JSON line for the reference arm, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    res = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, res.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["steps"] == 1
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0

