"""Expert parallelism across processes (include/ep_comm.h) on one B200.

The ranks are processes, each with its own CUDA context on the same GPU,
sharing their buffers through CUDA IPC; their barriers are host barriers
(EP_SYNC_HOST, over a gloo process group), so no kernel ever waits for
another process's kernel. Every rank compares its receive rows, meta
records, count and output rows with the CPU oracle of the whole W-rank
problem, bit for bit. EP_SYNC_DEVICE, whose barrier kernels wait for the
other ranks' kernels, needs a GPU per rank; here it runs as a single rank
(its barrier with itself), and a two-rank communicator on one GPU must be
refused.
"""
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import combine_ep_dispatch_05_b200 as ep  # noqa: E402
import comm_harness  # noqa: E402
from synth.inputs import workload  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _spawn(target, W, spec, extra=()):
    import torch.multiprocessing as tmp
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    args = [tuple(e(ctx) for e in extra)] if extra else [()]
    procs = [ctx.Process(target=target, args=(r, W, port, spec, q, *args[0])) for r in range(W)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(W):
            rank, status, data = q.get(timeout=600)
            got[rank] = (status, data)
    finally:
        for p in procs:
            p.join(timeout=120)
            if p.is_alive():
                p.kill()
    for r in range(W):
        assert got[r][0] == "ok", f"rank {r}: {got[r][0]}"
    return got


@pytest.mark.parametrize("W,spec", [
    (2, {"workload": "tiny", "seeds": [0, 5]}),
    (4, {"workload": "pr599", "replace": {"h": 1024}, "seeds": [1, 2]}),   # PR #599's shape, narrower rows
    (4, {"workload": "latency8", "replace": {"h": 512, "max_tok": 64, "max_recv": 256}, "seeds": [3]}),
    (3, {"workload": "skewed", "replace": {"h": 256, "max_tok": 300, "ct": 300, "max_recv": 900,
                                          "n_epr": 8}, "seeds": [4]}),  # hot destination, W not a power of 2
    (2, {"workload": "tiny", "replace": {"dtype": 1, "h": 64}, "seeds": [6]}),     # fp32 rows and combine
    (2, {"workload": "tiny", "replace": {"dtype": 2, "h": 256}, "seeds": [7]}),    # fp8 rows, bf16 combine
    (3, {"workload": "pr599", "replace": {"h": 1040}, "seeds": [8],                # the combine's 32-byte
         "env": {"EP_COMBINE_WIDE": "1"}}),                                          # loads, 2080-byte rows
    (2, {"workload": "tiny", "replace": {"dtype": 1, "h": 72}, "seeds": [9],       # and over fp32 rows
         "env": {"EP_COMBINE_WIDE": "1"}}),
])
def test_ranks_in_processes_match_the_oracle(W, spec):
    spec = dict(spec, sync=ep.EP_SYNC_HOST)
    got = _spawn(comm_harness.rank_main, W, spec)
    assert sum(got[r][1][0] for r in range(W)) > 0  # rows arrived somewhere


def test_rank_leaving_between_calls_is_reported():
    spec = {"workload": "tiny", "timeout_s": 5}
    _spawn(comm_harness.leaving_rank_main, 2, spec, extra=(lambda ctx: ctx.Event(),))


def _single_rank_comm(wl, sync=ep.EP_SYNC_DEVICE):
    comm = ep.ep_comm_create(wl.cfg(), 0, sync)
    ep.ep_comm_connect(comm, [ep.ep_comm_handle(comm)])
    return comm


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("pr599", {"h": 2048}), ("latency1", {})])
def test_device_sync_single_rank_matches_the_oracle(name, kw):
    wl = workload(name).replace(W=1, n_epr=workload(name).E, max_recv=0, **kw)
    comm = _single_rank_comm(wl)
    try:
        for seed in (wl.seed, wl.seed + 1):  # the device epoch advances across calls
            comm_harness.check_step(torch, ep, comm, wl.replace(seed=seed), 0)
        assert ep.ep_comm_check_error(comm) == 0
    finally:
        ep.ep_comm_destroy(comm)


def test_device_barrier_timeout_is_reported_and_the_context_survives(monkeypatch):
    """A barrier that no rank can complete (test hook): the wait gives up after
    about a second, EP_DEVERR_TIMEOUT is reported, the kernels after it write
    nothing, and the device keeps working."""
    monkeypatch.setenv("EP_TEST_UNREACHABLE_BARRIER", "1")
    wl = workload("tiny").replace(W=1, n_epr=8, max_recv=0)
    comm = _single_rank_comm(wl)
    try:
        from gpu_harness import as_bytes, to_dev
        from synth.inputs import make_inputs
        inputs = make_inputs(wl)
        info = ep.ep_comm_info(comm)
        recv_count = comm_harness.device_tensor(info.recvCount, (1,), "<i4")
        recv_count.fill_(-7)
        recv_x = comm_harness.device_tensor(info.recvX, (info.maxRecv, info.rowBytes), "|u1")
        recv_x.fill_(0xAB)
        ep.ep_comm_dispatch(comm, to_dev(as_bytes(inputs["x"][0])), to_dev(inputs["topk_idx"][0]),
                            to_dev(inputs["topk_w"][0]), torch.cuda.current_stream())
        assert ep.ep_comm_check_error(comm) & ep.EP_DEVERR_TIMEOUT
        assert int(recv_count.cpu()[0]) == -7 and bool((recv_x == 0xAB).all())  # nothing written
    finally:
        ep.ep_comm_destroy(comm)
    monkeypatch.delenv("EP_TEST_UNREACHABLE_BARRIER")
    from gpu_harness import run_and_compare
    from synth.inputs import make_inputs
    run, _ = run_and_compare(workload("tiny").cfg(), make_inputs(workload("tiny")))
    run.close()


def test_device_sync_refuses_two_ranks_on_one_gpu():
    wl = workload("tiny")
    comms = [ep.ep_comm_create(wl.cfg(), r, ep.EP_SYNC_DEVICE) for r in range(2)]
    try:
        recs = [ep.ep_comm_handle(c) for c in comms]
        with pytest.raises(ep.EpError) as e:
            ep.ep_comm_connect(comms[0], recs)
        assert e.value.code == ep.EP_ERR_UNSUPPORTED
    finally:
        for c in comms:
            ep.ep_comm_destroy(c)


def test_connect_refuses_mismatched_records():
    wl = workload("tiny")
    a = ep.ep_comm_create(wl.cfg(), 0, ep.EP_SYNC_HOST, barrier=lambda: None)
    b = ep.ep_comm_create(wl.replace(h=512).cfg(), 1, ep.EP_SYNC_HOST, barrier=lambda: None)
    try:
        with pytest.raises(ep.EpError) as e:
            ep.ep_comm_connect(a, [ep.ep_comm_handle(a), ep.ep_comm_handle(b)])
        assert e.value.code == ep.EP_ERR_INVALID
        with pytest.raises(ep.EpError):  # not in rank order
            ep.ep_comm_connect(a, [ep.ep_comm_handle(a), ep.ep_comm_handle(a)])
    finally:
        ep.ep_comm_destroy(a)
        ep.ep_comm_destroy(b)


@pytest.mark.parametrize("W", [2, 3, 8, 32])
def test_device_barrier_protocol_with_emulated_ranks(W):
    """The EP_SYNC_DEVICE barrier among W ranks, emulated by the W blocks of
    one cooperative launch on this GPU: every round completes on every rank,
    and what each rank wrote before a barrier is visible to all after it."""
    done, errs, early = ep.ep_comm_barrier_selftest(W, 200)
    assert done == [200] * W and errs == [0] * W and early == [0] * W


def test_device_barrier_gives_up_when_a_rank_stops_arriving():
    """Rank 1 stops arriving after its third barrier: the others pass 3
    barriers, then their wait gives up (about a second) with EP_DEVERR_TIMEOUT;
    no rank hangs."""
    done, errs, early = ep.ep_comm_barrier_selftest(4, 10, 1, 3)
    assert done == [3, 3, 3, 3] and early == [0] * 4
    assert errs[1] == 0 and all(errs[r] & ep.EP_DEVERR_TIMEOUT for r in (0, 2, 3))
    from gpu_harness import run_and_compare  # the device keeps working
    from synth.inputs import make_inputs
    run, _ = run_and_compare(workload("tiny").cfg(), make_inputs(workload("tiny")))
    run.close()


def test_device_sync_calls_replay_in_a_cuda_graph():
    """EP_SYNC_DEVICE calls do no host synchronisation, so they can be
    captured: a graph of dispatch + combine, replayed three times, gives the
    eager results each time (the barrier epoch advances on the device)."""
    wl = workload("pr599").replace(W=1, n_epr=32, max_recv=0, h=1024)
    comm = _single_rank_comm(wl)
    try:
        from gpu_harness import as_bytes, to_dev
        from synth.inputs import make_inputs
        inputs = make_inputs(wl)
        info = ep.ep_comm_info(comm)
        x = to_dev(as_bytes(inputs["x"][0]))
        idx = to_dev(inputs["topk_idx"][0])
        w = to_dev(inputs["topk_w"][0])
        recv_x = comm_harness.device_tensor(info.recvX, (info.maxRecv, info.rowBytes), "|u1")
        y = recv_x.view(torch.bfloat16).view(info.maxRecv, -1)
        out = torch.empty((wl.max_tok, wl.h), dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            ep.ep_comm_dispatch(comm, x, idx, w, s)
            ep.ep_comm_combine(comm, y, out, s)
        s.synchronize()
        eager = out.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                ep.ep_comm_dispatch(comm, x, idx, w, s)
                ep.ep_comm_combine(comm, y, out, s)
        for _ in range(3):
            out.fill_(0)
            g.replay()
            torch.cuda.synchronize()
            assert torch.equal(out, eager)
        assert ep.ep_comm_check_error(comm) == 0
        del g
    finally:
        ep.ep_comm_destroy(comm)
