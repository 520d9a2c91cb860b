"""ep_dispatch_noalloc against ep_dispatch, through the C ABI (needs a B200).

ep_dispatch_noalloc serves callers that cannot allocate device memory at the
point where they dispatch: a serving loop whose memory pool must not grow, code
running inside an allocator or driver callback (allocating there would re-enter
the allocator), or an embedder whose runtime owns every device allocation. Its
scratch is a fixed device array inside the library instead of a plan's
allocation.

Two calls in a row, on different routings and shapes, must each give exactly
(bit for bit, the bar every dispatch test here uses) the receive rows, meta
records and counts that a plan's ep_dispatch gives on the same inputs; a
configuration whose scratch would not fit the array must be refused with a
clear error. This file is collected last so that a run that stops at the first
failure has run everything else before it.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a CUDA device", allow_module_level=True)

import combine_ep_dispatch_05_b200 as ep  # noqa: E402
from synth.inputs import make_inputs, workload  # noqa: E402


def _buffers(wl, inputs):
    dev = torch.device("cuda")
    R = wl.max_recv
    return dict(
        x=torch.from_numpy(inputs["x"].view(np.int16)).to(dev),
        idx=torch.from_numpy(inputs["topk_idx"]).to(dev),
        w=None if inputs["topk_w"] is None else torch.from_numpy(inputs["topk_w"]).to(dev),
        recv_x=torch.full((wl.W, R, wl.h), -1, dtype=torch.int16, device=dev),
        recv_meta=torch.full((wl.W, R, 3 + wl.k), -1, dtype=torch.int32, device=dev),
        recv_count=torch.full((wl.W,), -1, dtype=torch.int32, device=dev),
    )


def _check_against_plan(wl):
    inputs = make_inputs(wl)
    cfg = wl.cfg()
    s = torch.cuda.current_stream()
    ref = _buffers(wl, inputs)
    plan = ep.ep_plan_create(cfg)
    try:
        ep.ep_dispatch(plan, ref["x"], ref["idx"], ref["w"], ref["recv_x"], ref["recv_meta"],
                       ref["recv_count"], s)
        torch.cuda.synchronize()
        assert ep.ep_plan_check_error(plan) == 0
    finally:
        ep.ep_plan_destroy(plan)
    got = _buffers(wl, inputs)
    ep.ep_dispatch_noalloc(cfg, got["x"], got["idx"], got["w"], got["recv_x"], got["recv_meta"],
                           got["recv_count"], s)
    torch.cuda.synchronize()
    assert torch.equal(got["recv_count"], ref["recv_count"])
    for pe in range(wl.W):
        n = int(ref["recv_count"][pe])
        assert torch.equal(got["recv_x"][pe, :n], ref["recv_x"][pe, :n]), pe
        assert torch.equal(got["recv_meta"][pe, :n], ref["recv_meta"][pe, :n]), pe
        assert bool((got["recv_x"][pe, n:] == -1).all())  # nothing written past the count


def test_noalloc_matches_plan_dispatch_two_calls():
    _check_against_plan(workload("pr599"))                 # first call on this device: set-up
    _check_against_plan(workload("main").replace(seed=9))  # second call: other shape, other routing


def test_noalloc_matches_plan_dispatch_on_sparse_and_unweighted_batches():
    """The call always scans the tile counts in route_count's last block and
    hands out tokens by the present-token total; plans take that form only
    under overrides. Batches with absent tokens (ct = 1 and 8 of 512 tokens a
    rank, no weights) and the tiny batch must still match a plan bit for bit."""
    for name in ("latency1", "latency8", "tiny"):
        _check_against_plan(workload(name))


def test_noalloc_refuses_configurations_beyond_its_scratch():
    cfg = dict(worldSize=32, hiddenDim=64, maxTokPerRank=1024, numExpertPerRank=2,
               numExpertPerToken=4, maxRecv=0, dtype=0, useWeights=0)
    one = torch.zeros(16, dtype=torch.int32, device="cuda")
    with pytest.raises(ep.EpError) as e:
        ep.ep_dispatch_noalloc(cfg, one, one, None, one, one, one, torch.cuda.current_stream())
    assert e.value.code == ep.EP_ERR_INVALID
    assert "scratch" in str(e.value)
