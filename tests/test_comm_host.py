"""Host side of expert parallelism across processes, without a GPU: the
connection records travel between gloo ranks in rank order, and the C ABI
rejects bad arguments before it touches a device."""
import ctypes
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        from combine_ep_dispatch_05_b200 import comm
        rec = bytes([rank]) * 256  # stands in for ep_comm_handle's record
        q.put((rank, comm.gather_records(rec, dist)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_records_reach_every_rank_in_rank_order():
    import torch.multiprocessing as tmp
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 3
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert [rec[0] for rec in got[r]] == list(range(world))
        assert all(len(rec) == 256 for rec in got[r])


@pytest.fixture(scope="module")
def binding():
    from combine_ep_dispatch_05_b200 import build
    build.build()
    from combine_ep_dispatch_05_b200 import binding as b
    return b


def _cfg(b, **kw):
    c = dict(worldSize=2, hiddenDim=256, maxTokPerRank=8, numExpertPerRank=4, numExpertPerToken=2,
             maxRecv=0, dtype=0, useWeights=1)
    c.update(kw)
    return b._cfg(c)


@pytest.mark.parametrize("rank,sync,with_barrier", [(2, 0, False), (-1, 0, False), (0, 7, False), (0, 1, False)])
def test_create_rejects_bad_arguments_before_the_device(binding, rank, sync, with_barrier):
    cfg = _cfg(binding)
    h = binding._lib.ep_comm_create(ctypes.byref(cfg), rank, sync, binding.HOST_BARRIER(), None)
    assert not h
    msg = binding.ep_last_error()
    assert "rank" in msg or "sync" in msg or "barrier" in msg


def test_create_rejects_invalid_configuration(binding):
    h = binding._lib.ep_comm_create(ctypes.byref(_cfg(binding, hiddenDim=7)), 0, 0, binding.HOST_BARRIER(), None)
    assert not h and "multiple of 16" in binding.ep_last_error()


def test_entry_points_reject_null(binding):
    lib = binding._lib
    assert lib.ep_comm_dispatch(None, None, None, None, None) == binding.EP_ERR_INVALID
    assert lib.ep_comm_combine(None, None, None, None) == binding.EP_ERR_INVALID
    assert lib.ep_comm_handle(None, None) == binding.EP_ERR_INVALID
    assert lib.ep_comm_connect(None, None) == binding.EP_ERR_INVALID
    assert lib.ep_comm_info(None, None) == binding.EP_ERR_INVALID
    assert lib.ep_comm_check_error(None) == binding.EP_ERR_INVALID
    lib.ep_comm_destroy(None)


def test_create_without_a_device_fails_cleanly(binding):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(binding.EpError) as e:
        binding.ep_comm_create(_cfg(binding), 0, binding.EP_SYNC_DEVICE)
    assert "cuda" in str(e.value).lower() or "device" in str(e.value).lower()
