"""bench.py's multi-rank path (the communicator under torchrun) on the one
GPU here: EP_BENCH_SHARE_GPU=1 puts both ranks on GPU 0 with host barriers
and a gloo process group. The bench checks its own step (received-row count
against every rank's routing, output rows against row times weight sum)
before it times, and prints one JSON line."""
import json
import os
import socket
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_bench_runs_two_ranks_sharing_one_gpu():
    env = dict(os.environ, EP_BENCH_SHARE_GPU="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
           "--steps", "3", "--warmup", "2", "--workload", "pr599"]
    out = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-3000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["n_gpus"] == 2 and line["config"]["world_size"] == 2
    assert "host barriers" in line["config"]["parallelism"]
    assert line["value"] > 0 and line["dispatch_us"] > 0 and line["combine_us"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] > 0 and line["gpu_launches"] == 7 * 3


def test_bench_runs_the_device_barrier_path_with_one_rank():
    """EP_BENCH_COMM=1 under torchrun with one rank: the path a multi-GPU run
    takes (device barriers, NCCL process group and all-to-allv baseline,
    self-check, end-to-end timing), with W = 1."""
    env = dict(os.environ, EP_BENCH_COMM="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=1",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "1",
           "--steps", "3", "--warmup", "2", "--workload", "pr599"]
    out = subprocess.run(cmd, env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-3000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["n_gpus"] == 1 and line["config"]["world_size"] == 1
    assert "device barriers" in line["config"]["parallelism"]
    assert line["nccl_baseline"]["step_us"] > 0 and line["value"] > 0
