"""The bench's multi-process host logic on CPU: two gloo ranks.

With N GPUs the bench runs N replicas (each GPU holds all W virtual ranks). The
host side of that path is the rank setup from the launcher's environment and
the max-over-ranks reduction of the timings; the reference arm runs on rank 0
only. These need no GPU and run here with the gloo backend.
"""
import json
import os
import socket
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        r, w, local, d = bench.dist_setup(world)
        got = bench.max_over_ranks(1.5 * (rank + 1), d, "cpu")
        q.put((rank, r, w, local, got))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks():
    import torch.multiprocessing as tmp
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[0] for o in out] == [0, 1]
    for rank, r, w, local, got in out:
        assert (r, w, local) == (rank, 2, rank)
        assert got == pytest.approx(3.0)  # every rank sees the slowest rank's time


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    wl = bench.get_workload("tiny")
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, impl="reference", workload="tiny")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("LOCAL_RANK", "1")
    assert bench.run_reference(args, wl) == 0
    assert capsys.readouterr().out == ""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("LOCAL_RANK", "0")
    assert bench.run_reference(args, wl) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "us" and line["higher_is_better"] is False
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] == line["value"]
    assert cpu["cores"] >= 1 and cpu["nproc"] >= 1 and cpu["cpu_model"]
    assert cpu["single_core_us"] > 0 and "full tiny workload" in cpu["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0


def _nccl_baseline_worker(rank, world, port, q):
    """The bench's all-to-allv baseline on gloo ranks (CPU tensors): its
    received rows are the oracle's, in the same (source rank, token) order,
    and its output rows are within the spec's tolerance of the oracle's."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import numpy as np
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import oracle
        wl = bench.comm_workload(bench.get_workload("tiny").replace(h=64, max_tok=16, ct=12), world)
        parts = [bench.rank_inputs(wl, r) for r in range(world)]
        full = {k: np.stack([p[k] for p in parts]) for k in ("x", "topk_idx", "topk_w")}
        ref = oracle.dispatch(wl.cfg(), full["x"], full["topk_idx"], full["topk_w"])
        ref_out = oracle.combine(wl.cfg(), ref["recv_x"], ref["slotmap"], ref["wsum"])
        mine = parts[rank]
        x = torch.from_numpy(mine["x"].view(np.uint8).reshape(wl.max_tok, -1))
        out, recv = bench.nccl_alltoallv_step(x, torch.from_numpy(mine["topk_idx"]),
                                             torch.from_numpy(mine["topk_w"]), world, wl.n_epr, dist)
        n = int(ref["recv_count"][rank])
        ok_rows = recv.shape[0] == n and np.array_equal(recv.numpy().view(np.uint16).reshape(n, -1),
                                                         ref["recv_x"][rank, :n])
        got = out.float().numpy()
        exp = torch.from_numpy(ref_out[rank].view(np.int16)).view(torch.bfloat16).float().numpy()
        ok_out = bool((np.abs(got - exp) <= 2.0 ** -7 * np.abs(exp) + 1e-3).all())
        q.put((rank, ok_rows, ok_out))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_nccl_baseline_logic_on_gloo():
    import torch.multiprocessing as tmp
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_nccl_baseline_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_rows, ok_out in got:
        assert ok_rows, f"rank {rank}: received rows differ from the oracle's"
        assert ok_out, f"rank {rank}: output outside tolerance"


def test_comm_workload_keeps_the_expert_count():
    sys.path.insert(0, ROOT)
    import bench
    wl = bench.get_workload("main")
    for n in (1, 2, 4, 8):
        c = bench.comm_workload(wl, n)
        assert c.W == n and c.E == wl.E and c.max_recv == n * wl.max_tok and c.max_tok == wl.max_tok
