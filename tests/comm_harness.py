"""Ranks of a communicator (include/ep_comm.h) as processes for the tests.

Each rank is a process started with the spawn method (CUDA must not be
initialised before a fork). The ranks meet through a gloo process group: it
carries the connection records (an all-gather) and serves as the host
barrier of EP_SYNC_HOST. Every rank checks its own results against the CPU
oracle of the whole W-rank problem (dispatch outputs bit for bit, combine bit
for bit and within the spec's tolerance) and reports "ok" or the failure on a
queue.
"""
from __future__ import annotations

import os
import sys
import traceback
from datetime import timedelta

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class DeviceMemory:
    """A view of device memory the library owns, for torch.as_tensor."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def device_tensor(ptr, shape, typestr):
    import torch
    return torch.as_tensor(DeviceMemory(ptr, shape, typestr), device="cuda")


def _setup(rank, W, port, timeout_s):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    for p in (ROOT, os.path.join(ROOT, "tests")):
        if p not in sys.path:
            sys.path.insert(0, p)
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=W, timeout=timedelta(seconds=timeout_s))
    return torch, dist


def _connect(ep, dist, cfg, rank, W, sync):
    comm = ep.ep_comm_create(cfg, rank, sync, barrier=dist.barrier if sync == ep.EP_SYNC_HOST else None)
    recs = [None] * W
    dist.all_gather_object(recs, ep.ep_comm_handle(comm))
    ep.ep_comm_connect(comm, recs)
    return comm


def check_step(torch, ep, comm, wl, rank):
    """One dispatch + combine of this rank, compared with the oracle."""
    import oracle
    from gpu_harness import as_bytes, combine_torch_dtype, random_combine_input, to_dev
    cfg = wl.cfg()
    from synth.inputs import make_inputs
    inputs = make_inputs(wl)
    ref = oracle.dispatch(cfg, inputs["x"], inputs["topk_idx"], inputs["topk_w"])
    byte_payload = wl.dtype in (2, 3)
    y_full = random_combine_input(cfg, seed=wl.seed + 77) if byte_payload else ref["recv_x"]
    ref_out = oracle.combine(cfg, y_full, ref["slotmap"], ref["wsum"])

    info = ep.ep_comm_info(comm)
    R, row, M, T = info.maxRecv, info.rowBytes, info.metaFields, wl.max_tok
    hc = info.combineRowBytes // (4 if wl.dtype == 1 else 2)
    x = to_dev(as_bytes(inputs["x"][rank]))
    idx = to_dev(inputs["topk_idx"][rank])
    w = None if inputs["topk_w"] is None else to_dev(inputs["topk_w"][rank])
    recv_x = device_tensor(info.recvX, (R, row), "|u1")
    recv_meta = device_tensor(info.recvMeta, (R, M), "<i4")
    recv_count = device_tensor(info.recvCount, (1,), "<i4")
    recv_x.fill_(0xAB)  # canary past the count
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    ep.ep_comm_dispatch(comm, x, idx, w, s)
    torch.cuda.synchronize()
    n = int(recv_count.cpu()[0])
    assert n == int(ref["recv_count"][rank]), (n, ref["recv_count"])
    ref_x = as_bytes(ref["recv_x"])[rank, :n]
    assert torch.equal(recv_x[:n], torch.from_numpy(ref_x).cuda()), "receive rows differ"
    assert bool((recv_x[n:] == 0xAB).all()), "receive rows written past the count"
    assert torch.equal(recv_meta[:n], torch.from_numpy(ref["recv_meta"][rank, :n]).cuda()), "meta differs"

    ct = combine_torch_dtype(cfg)
    if byte_payload:
        y = to_dev(np.ascontiguousarray(y_full[rank])).view(ct)
    else:
        y = recv_x.view(ct).view(R, hc)
    out = torch.empty((T, hc), dtype=ct, device="cuda")
    out.view(torch.int16).fill_(0x7FC1)  # canary: every row must be written
    ep.ep_comm_combine(comm, y, out, s)
    torch.cuda.synchronize()
    ro = np.ascontiguousarray(ref_out[rank])
    if wl.dtype == 1:
        assert torch.equal(out.view(torch.int32), torch.from_numpy(ro.view(np.int32)).cuda()), "combine differs"
    else:
        got = out.view(torch.bfloat16).float()
        refo = torch.from_numpy(ro.view(np.int16)).cuda().view(torch.bfloat16).float()
        assert bool(((got - refo).abs() <= 2.0 ** -7 * refo.abs() + 1e-3).all()), "combine outside tolerance"
        assert torch.equal(out.view(torch.int16), torch.from_numpy(ro.view(np.int16)).cuda()), \
            "combine not bit-exact"
    return n


def rank_main(rank, W, port, spec, q):
    """spec: {"workload": name, "replace": {...}, "seeds": [...], "sync": 0|1,
    "env": {...} (optional: environment of the library in this rank)}.
    Runs one step per seed on one communicator."""
    try:
        os.environ.update(spec.get("env", {}))
        torch, dist = _setup(rank, W, port, spec.get("timeout_s", 60))
        import combine_ep_dispatch_05_b200 as ep
        from synth.inputs import workload
        base = workload(spec["workload"]).replace(W=W, **spec.get("replace", {}))
        comm = _connect(ep, dist, base.cfg(), rank, W, spec["sync"])
        counts = []
        for seed in spec["seeds"]:
            counts.append(check_step(torch, ep, comm, base.replace(seed=seed), rank))
        assert ep.ep_comm_check_error(comm) == 0
        dist.barrier()  # no rank frees its memory while another may still use it
        ep.ep_comm_destroy(comm)
        q.put((rank, "ok", counts))
    except BaseException:
        q.put((rank, "FAIL\n" + traceback.format_exc(), None))


def leaving_rank_main(rank, W, port, spec, q, release):
    """Both ranks run one checked step; then rank 1 stops making calls (it
    stays alive, holding its memory, until rank 0 releases it). Rank 0's next
    dispatch must fail with EP_ERR_PEER at its start barrier, without a kernel
    touching rank 1, and this process must still be able to run a plan's
    dispatch and combine correctly."""
    try:
        torch, dist = _setup(rank, W, port, spec.get("timeout_s", 5))
        import combine_ep_dispatch_05_b200 as ep
        from synth.inputs import make_inputs, workload
        base = workload(spec["workload"]).replace(W=W, **spec.get("replace", {}))
        comm = _connect(ep, dist, base.cfg(), rank, W, ep.EP_SYNC_HOST)
        check_step(torch, ep, comm, base, rank)
        if rank == 1:
            release.wait(120)  # gone from the communicator, memory still mapped by rank 0
            ep.ep_comm_destroy(comm)
            q.put((rank, "ok", None))
            return
        inputs = make_inputs(base)
        from gpu_harness import as_bytes, run_and_compare, to_dev
        x = to_dev(as_bytes(inputs["x"][rank]))
        idx = to_dev(inputs["topk_idx"][rank])
        w = None if inputs["topk_w"] is None else to_dev(inputs["topk_w"][rank])
        try:
            ep.ep_comm_dispatch(comm, x, idx, w, torch.cuda.current_stream())
            raise AssertionError("dispatch without the other rank did not fail")
        except ep.EpError as e:
            assert e.code == ep.EP_ERR_PEER, e
        assert ep.ep_comm_check_error(comm) == 0  # no kernel ran into trouble
        ep.ep_comm_destroy(comm)
        release.set()
        # The context is still usable: a plan's dispatch and combine on one GPU.
        wl = workload("pr599").replace(h=512)
        run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
        run.close()
        q.put((rank, "ok", None))
    except BaseException:
        release.set()
        q.put((rank, "FAIL\n" + traceback.format_exc(), None))
