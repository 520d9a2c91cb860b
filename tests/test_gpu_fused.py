"""The fused dispatch (EP_DISPATCH_FUSED=1: one launch; every block routes
its own share of the batch, adds up the earlier blocks' published totals and
copies its own tokens) against the CPU oracle, through the C ABI (needs a
B200).

The same bar as test_gpu_parity: dispatch bit-exact, rows and records past
recv_count keep their canaries, combine bit-exact with the oracle's fold.
Every case below that the per-block token bound admits takes this dispatch.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import combine_ep_dispatch_05_b200 as ep  # noqa: E402
import oracle  # noqa: E402
import oracle_pins as P  # noqa: E402
from gpu_harness import (CANARY_META, DeviceRun, compare_combine, compare_dispatch, run_and_compare,  # noqa: E402
                         to_dev)
from synth.inputs import make_inputs, workload  # noqa: E402

FUSED_MAX_OWN = 64  # tokens a block may own (kFusedMaxOwn)


@pytest.fixture(autouse=True)
def _fused(monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_FUSED", "1")


def _expect_fused(info, G, k=None):
    blocks = info.scatterBlocks
    if -(-G // min(blocks, G)) <= FUSED_MAX_OWN:
        assert info.dispatchFused == 1
        assert blocks <= G


@pytest.mark.parametrize("name", ["tiny", "pr599", "latency1", "latency8"])
def test_fused_workloads(name):
    wl = workload(name)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    assert run.info.dispatchFused == 1
    run.close()


@pytest.mark.parametrize("ct,topk", [(512, 6), (512, 8), (1024, 6), (2048, 8), (1, 6), (8, 6)])
def test_fused_pr599_matrix(ct, topk):
    """mori PR #599's correctness matrix ("Perf/ep disp 1250 ship",
    correctness section) at the sizes this dispatch takes."""
    max_tok = max(ct, 512)
    wl = workload("pr599").replace(h=2048, ct=ct, max_tok=max_tok, max_recv=4 * max_tok, k=topk,
                                   seed=2000 + ct + topk)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    _expect_fused(run.info, wl.W * wl.max_tok, wl.k)
    run.close()


@pytest.mark.parametrize("case", [
    # W, T, h, k, nEpr, weights, maxRecv
    (3, 300, 264, 5, 3, True, 0),       # 528-byte rows, chunks straddling block ranges
    (1, 513, 128, 4, 6, True, 0),       # single rank
    (32, 9, 64, 32, 2, True, 0),        # max world size and max topk
    (5, 77, 8, 7, 1, False, 500),       # 16-byte rows, maxRecv above W*T, no weights
    (2, 40, 20000, 3, 4, True, 0),      # 40000-byte rows: copied in three pieces
    (8, 1000, 1024, 6, 8, True, 0),     # 55 tokens a block
    (7, 3, 256, 3, 3, True, 0),         # fewer tokens than blocks
    (16, 100, 512, 16, 3, True, 0),     # topk 16 (second ids instance), nEpr not a power of two
    (32, 296, 64, 32, 1, True, 0),      # 9472 tokens: 64 a block, W = k = 32, the largest routing area
])
def test_fused_random(case):
    W, T, h, k, nEpr, use_w, max_recv = case
    rng = np.random.default_rng(hash(case) % (1 << 32))
    E = W * nEpr
    idx = rng.integers(-2, E, size=(W, T, k)).astype(np.int32)
    xb = P.torch_bf16_bits(rng.standard_normal((W, T, h)).astype(np.float32))
    w = rng.standard_normal((W, T, k)).astype(np.float32) if use_w else None
    cfg = dict(worldSize=W, hiddenDim=h, maxTokPerRank=T, numExpertPerRank=nEpr,
               numExpertPerToken=k, maxRecv=max_recv, dtype=0, useWeights=int(use_w))
    run, _ = run_and_compare(cfg, dict(x=xb, topk_idx=idx, topk_w=w))
    _expect_fused(run.info, W * T, k)
    run.close()


@pytest.mark.parametrize("dtype", [0, 1, 2, 3], ids=["bf16", "fp32", "fp8", "fp4x2"])
def test_fused_dtype_random_small(dtype):
    rng = np.random.default_rng(300 + dtype)
    for _ in range(6):
        cfg, xb, idx, w = P.random_small_case(rng, dtype=dtype)
        run, _ = run_and_compare(cfg, dict(x=xb, topk_idx=idx, topk_w=w))
        assert run.info.dispatchFused == 1
        run.close()


def test_fused_scaled():
    """Scale rows travel with the payload (ep_dispatch_scaled)."""
    rng = np.random.default_rng(41)
    for case in range(6):
        cfg, xb, idx, w = P.random_small_case(rng, dtype=case % 4)
        sw = int(rng.integers(1, 80))
        W, T = cfg["worldSize"], cfg["maxTokPerRank"]
        scales = rng.standard_normal((W, T, sw)).astype(np.float32)
        ref = oracle.dispatch(cfg, xb, idx, w, scales=scales)
        with DeviceRun(cfg, dict(x=xb, topk_idx=idx, topk_w=w)) as run:
            assert run.info.dispatchFused == 1
            R = run.info.maxRecv
            rs = torch.full((W, R, sw), 0x0C0FFEE, dtype=torch.int32, device="cuda")
            ep.ep_dispatch_scaled(run.plan, run.x, run.idx, run.w, to_dev(scales), sw, run.recv_x,
                                  run.recv_meta, rs, run.recv_count, torch.cuda.current_stream())
            torch.cuda.synchronize()
            compare_dispatch(run, ref)
            ref_s = torch.from_numpy(ref["recv_scales"].view(np.int32)).to("cuda")
            for pe in range(W):
                n = int(ref["recv_count"][pe])
                assert torch.equal(rs[pe, :n], ref_s[pe, :n])
                assert bool((rs[pe, n:] == 0x0C0FFEE).all())
            assert run.error_word() == 0


def test_fused_out_of_range_ids():
    rng = np.random.default_rng(5)
    W, T, k, nEpr = 4, 64, 4, 4
    idx = rng.integers(-2, W * nEpr + 3, size=(W, T, k)).astype(np.int32)
    assert (idx >= W * nEpr).any()
    xb = P.torch_bf16_bits(rng.standard_normal((W, T, 64)).astype(np.float32))
    w = rng.standard_normal((W, T, k)).astype(np.float32)
    cfg = dict(worldSize=W, hiddenDim=64, maxTokPerRank=T, numExpertPerRank=nEpr,
               numExpertPerToken=k, maxRecv=0, dtype=0, useWeights=1)
    run, ref = run_and_compare(cfg, dict(x=xb, topk_idx=idx, topk_w=w))
    assert ref["status"] == oracle.STATUS_EXPERT_RANGE
    run.close()


def test_fused_empty_call():
    wl = workload("latency1")
    inputs = make_inputs(wl)
    inputs["topk_idx"][:] = -1
    run, ref = run_and_compare(wl.cfg(), inputs)
    assert int(ref["recv_count"].sum()) == 0
    assert bool((run.out == 0).all())
    run.close()


def test_fused_repeated_calls_and_graph():
    """Two routings on one plan, then dispatch + combine captured in a CUDA
    graph and replayed: every replay matches the eager results."""
    wl = workload("pr599").replace(h=512)
    cfg = wl.cfg()
    a = make_inputs(wl)
    b = make_inputs(wl.replace(seed=78))
    ref_b = oracle.dispatch(cfg, b["x"], b["topk_idx"], b["topk_w"])
    run, _ = run_and_compare(cfg, a)
    run.load_inputs(b)
    run.reset_canaries()
    run.dispatch()
    run.combine()
    torch.cuda.synchronize()
    compare_dispatch(run, ref_b)
    compare_combine(run, oracle.combine(cfg, ref_b["recv_x"], ref_b["slotmap"], ref_b["wsum"]))
    eager_out = run.out.clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            run.dispatch(stream=s)
            run.combine(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        run.out.fill_(0x7FC1)
        run.recv_count.fill_(-7)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(run.out, eager_out)
        assert np.array_equal(run.recv_count.cpu().numpy(), ref_b["recv_count"])
    assert run.error_word() == 0
    del g
    run.close()


@pytest.mark.parametrize("env", [
    {"EP_SCATTER_STAGES": "2"},
    {"EP_SCATTER_STAGES": "4", "EP_SCATTER_CHUNK": "4096"},  # rows in pieces
    {"EP_SCATTER_WARPS": "1"},                               # one engine, seven routing warps
    {"EP_SCATTER_WARPS": "8", "EP_SCATTER_STAGES": "2", "EP_SCATTER_CHUNK": "1024"},  # every warp an engine
    {"EP_SCATTER_BLOCKS": "40"},                             # 52 tokens a block
    {"EP_SCATTER_BLOCKS": "31"},                             # 67 a block: over the bound, split dispatch
])
def test_fused_geometry(env, monkeypatch):
    for k_, v in env.items():
        monkeypatch.setenv(k_, v)
    wl = workload("pr599").replace(h=1536)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    G = wl.W * wl.max_tok
    if env.get("EP_SCATTER_BLOCKS") == "31":
        assert run.info.dispatchFused == 0
    else:
        _expect_fused(run.info, G, wl.k)
    run.close()


def test_fused_lookback_wait_runs_out(monkeypatch):
    """Failure detection without a GPU fault: the test hook makes every block
    wait for a tag that no block publishes. Block 0, which waits on nothing,
    copies its own tokens; every other block gives up after its bounded wait
    and copies nothing. The host reads EP_DEVERR_TIMEOUT, and a fresh plan on
    the same context works."""
    monkeypatch.setenv("EP_TEST_UNREACHABLE_BARRIER", "1")
    wl = workload("latency8")
    inputs = make_inputs(wl)
    with DeviceRun(wl.cfg(), inputs) as run:
        assert run.info.dispatchFused == 1
        run.dispatch()
        err = run.error_word()  # synchronises: the kernel has returned
        assert err & ep.EP_DEVERR_TIMEOUT
        G = wl.W * wl.max_tok
        hi0 = G // run.info.scatterBlocks  # block 0 owns tokens [0, hi0), all of source rank 0
        assert 0 < hi0 <= wl.max_tok
        ref = oracle.dispatch(wl.cfg(), inputs["x"], inputs["topk_idx"], inputs["topk_w"])
        meta = run.recv_meta.cpu().numpy()
        rx = run.recv_x.cpu().numpy()
        for pe in range(wl.W):
            rm = ref["recv_meta"][pe]
            n0 = int(((rm[:, 0] == 0) & (rm[:, 1] < hi0) &
                      (np.arange(rm.shape[0]) < ref["recv_count"][pe])).sum())
            assert np.array_equal(meta[pe, :n0], rm[:n0])
            assert (meta[pe, n0:] == CANARY_META).all()
            assert np.array_equal(rx[pe, :n0], ref["recv_x"][pe, :n0].view(np.uint8).reshape(n0, -1))
            assert (rx[pe, n0:] == 0xAB).all()
    monkeypatch.delenv("EP_TEST_UNREACHABLE_BARRIER")
    run, _ = run_and_compare(wl.cfg(), inputs)  # the device is healthy
    run.close()
