"""CUDA path vs the CPU oracle, through the C ABI (needs a B200).

Dispatch outputs (recv_x, recv_meta, recv_count) must be bit-exact; rows and
records past recv_count must keep their canary; combine must be within
2^-7|oracle| + 1e-3 and, with the same fold order and one rounding per term,
bit-exact.
"""
import os

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # pragma: no cover - collected on CPU machines too
    pytest.skip("needs a CUDA device", allow_module_level=True)

import combine_ep_dispatch_05_b200 as ep  # noqa: E402
import oracle  # noqa: E402
import oracle_pins as P  # noqa: E402
from gpu_harness import (DeviceRun, compare_combine, compare_dispatch, run_and_compare,  # noqa: E402
                         to_dev)
from synth.inputs import WORKLOADS, make_inputs, workload  # noqa: E402


FUSED_MAX_OWN = 64  # tokens a block of the fused dispatch may own (kFusedMaxOwn)


def _fused_expected(info, fused, G):
    """EP_DISPATCH_FUSED=1 takes the one-launch dispatch when no block owns
    more than FUSED_MAX_OWN tokens."""
    if fused == "1" and info.dispatchFused:
        assert -(-G // info.scatterBlocks) <= FUSED_MAX_OWN
    return fused == "1" and -(-G // min(info.scatterBlocks, G)) <= FUSED_MAX_OWN


def test_library_is_in_tree():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    assert ep.library_path().startswith(root)


@pytest.mark.parametrize("name", ["tiny", "pr599", "latency1", "latency8", "main", "skewed"])
def test_workload_parity(name):
    wl = workload(name)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    run.close()


@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
@pytest.mark.parametrize("name", ["tiny", "pr599", "latency1", "latency8", "main"])
def test_workload_parity_both_dispatch_modes(name, fused, monkeypatch):
    """The workloads through both dispatch forms: route_count + scatter_rows,
    and the one-launch fused dispatch (which main, at 222 tokens a block, does
    not take)."""
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    wl = workload(name)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    assert run.info.dispatchFused == _fused_expected(run.info, fused, wl.W * wl.max_tok)
    assert run.info.dispatchFused == (fused == "1" and name != "main")
    run.close()


@pytest.mark.parametrize("dense", ["0", "1"], ids=["small-batch-form", "large-batch-form"])
@pytest.mark.parametrize("ct,topk", [(512, 6), (512, 8), (1024, 6), (1024, 8), (2048, 6), (2048, 8),
                                     (4096, 6), (4096, 8), (1, 6), (8, 6)])
def test_pr599_correctness_matrix(ct, topk, dense, monkeypatch):
    """The correctness matrix of mori PR #599 ("Perf/ep disp 1250 ship",
    correctness section): tokens per rank 512..4096 at topk 6 and 8 (topk 8
    reaches the paths with more than one entry per lane), and 1 or 8 live
    tokens of 512 at topk 6 (idle warps), at its EP4 shape with 8 experts per
    rank (hidden 2048 here: the row width is not what the matrix varies),
    through both forms of the split dispatch."""
    monkeypatch.setenv("EP_DISPATCH_DENSE", dense)
    max_tok = max(ct, 512)
    wl = workload("pr599").replace(h=2048, ct=ct, max_tok=max_tok, max_recv=4 * max_tok, k=topk,
                                   seed=1000 + ct + topk)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    run.close()


@pytest.mark.parametrize("name", ["main", "skewed"])
def test_large_batch_with_sparse_machinery(name, monkeypatch):
    """The main shapes through the small-batch form of the split dispatch
    (present-token column, scatter-side scan of the tile counts)."""
    monkeypatch.setenv("EP_DISPATCH_DENSE", "0")
    wl = workload(name)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    run.close()


def _small_random_cfg(rng, W, T, h, k, nEpr, use_w, max_recv=0, dup=True, oob=False):
    E = W * nEpr
    lo = -2 if dup else 0
    hi = E + (3 if oob else 0)
    idx = rng.integers(lo, hi, size=(W, T, k)).astype(np.int32)
    xb = P.torch_bf16_bits(rng.standard_normal((W, T, h)).astype(np.float32))
    w = rng.standard_normal((W, T, k)).astype(np.float32) if use_w else None
    cfg = dict(worldSize=W, hiddenDim=h, maxTokPerRank=T, numExpertPerRank=nEpr,
               numExpertPerToken=k, maxRecv=max_recv, dtype=0, useWeights=int(use_w))
    return cfg, dict(x=xb, topk_idx=idx, topk_w=w)


@pytest.mark.parametrize("case", [
    # W, T, h, k, nEpr, weights, maxRecv -- several routing tiles with a ragged tail
    (3, 300, 264, 5, 3, True, 0),       # 528-byte rows: combine column tail
    (1, 513, 128, 4, 6, True, 0),       # single rank
    (32, 9, 64, 32, 2, True, 0),        # max world size and max topk: 35 meta fields
    (5, 77, 8, 7, 1, False, 500),       # 16-byte rows, maxRecv above W*T, no weights
    (2, 40, 20000, 3, 4, True, 0),      # 40000-byte rows: copied in three pieces
    (8, 1000, 1024, 6, 8, True, 0),     # 4 tiles, ragged
])
@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
def test_random_parity(case, fused, monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    W, T, h, k, nEpr, use_w, max_recv = case
    rng = np.random.default_rng(hash(case) % (1 << 32))
    cfg, inputs = _small_random_cfg(rng, W, T, h, k, nEpr, use_w, max_recv)
    run, _ = run_and_compare(cfg, inputs)
    assert run.info.dispatchFused == _fused_expected(run.info, fused, W * T)
    run.close()


@pytest.mark.parametrize("dtype,h", [(1, 1024), (2, 1024), (3, 512)], ids=["fp32", "fp8", "fp4x2"])
def test_dtype_parity(dtype, h):
    """Narrow and wide payloads (design page §3.7): dispatch moves the payload
    bit for bit; the combine leg is fp32 for fp32 plans and bf16 otherwise (over
    2*h elements for fp4x2), here on a seeded expert output."""
    wl = workload("pr599").replace(dtype=dtype, h=h)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    assert run.info.rowBytes == h * {1: 4, 2: 1, 3: 1}[dtype]
    run.close()


@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
@pytest.mark.parametrize("dtype", [0, 1, 2, 3], ids=["bf16", "fp32", "fp8", "fp4x2"])
def test_dtype_random_small(dtype, fused, monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    """Arbitrary payload bits (NaN and inf patterns included for fp32), duplicate
    ids, masked entries, maxRecv above W*T."""
    rng = np.random.default_rng(100 + dtype)
    for _ in range(6):
        cfg, xb, idx, w = P.random_small_case(rng, dtype=dtype)
        run, _ = run_and_compare(cfg, dict(x=xb, topk_idx=idx, topk_w=w))
        run.close()


@pytest.mark.parametrize("case", [
    # W, T, h, k, nEpr, weights, maxRecv -- combine rows a multiple of 32 bytes
    (3, 300, 272, 5, 3, True, 0),       # 544-byte rows: 17 loads a row, a partial warp
    (8, 1000, 1024, 6, 8, True, 0),     # 4 tiles, ragged
    (2, 40, 20000, 3, 4, True, 0),      # 40000-byte rows
    (5, 77, 16, 7, 1, False, 500),      # one 32-byte load a row, no weights
])
def test_wide_combine_parity(case, monkeypatch):
    """The combine's 32-byte loads, forced on small plans (EP_COMBINE_WIDE=1):
    bit-exact against the oracle like the 16-byte loads."""
    monkeypatch.setenv("EP_COMBINE_WIDE", "1")
    W, T, h, k, nEpr, use_w, max_recv = case
    rng = np.random.default_rng(hash(case) % (1 << 32))
    cfg, inputs = _small_random_cfg(rng, W, T, h, k, nEpr, use_w, max_recv)
    run, _ = run_and_compare(cfg, inputs)
    assert run.info.combineLoadBytes == 32
    run.close()


@pytest.mark.parametrize("dtype", [1, 2, 3], ids=["fp32", "fp8", "fp4x2"])
def test_wide_combine_dtypes_random_small(dtype, monkeypatch):
    """32-byte combine loads over the other combine legs: fp32 (arbitrary bits,
    NaN and inf included) and the bf16 leg of byte payloads."""
    monkeypatch.setenv("EP_COMBINE_WIDE", "1")
    rng = np.random.default_rng(300 + dtype)
    wide = 0
    for _ in range(8):
        cfg, xb, idx, w = P.random_small_case(rng, dtype=dtype)
        run, _ = run_and_compare(cfg, dict(x=xb, topk_idx=idx, topk_w=w))
        wide += run.info.combineLoadBytes == 32
        run.close()
    assert wide > 0


def test_wide_combine_misaligned_y_takes_narrow_loads(monkeypatch):
    """A plan with 32-byte combine loads, called with a y that is 16- but not
    32-byte aligned: the call takes the 16-byte loads, with the same results."""
    monkeypatch.setenv("EP_COMBINE_WIDE", "1")
    wl = workload("pr599").replace(h=1024)
    cfg = wl.cfg()
    inputs = make_inputs(wl)
    run, ref = run_and_compare(cfg, inputs)
    assert run.info.combineLoadBytes == 32
    y = run.identity_y()
    n = y.numel() * y.element_size()
    buf = torch.empty(n + 64, dtype=torch.uint8, device="cuda")
    off = (16 - buf.data_ptr() % 32) % 32  # the first 16- but not 32-byte aligned offset
    yv = buf[off:off + n]
    assert yv.data_ptr() % 32 == 16
    yv.copy_(y.reshape(-1).view(torch.uint8))
    run.reset_canaries()
    run.dispatch()
    run.combine(y=yv.view(y.dtype).view(y.shape))
    torch.cuda.synchronize()
    compare_combine(run, oracle.combine(cfg, ref["recv_x"], ref["slotmap"], ref["wsum"]))
    assert run.error_word() == 0
    run.close()


@pytest.mark.parametrize("dtype,h", [(2, 7168), (3, 3584)], ids=["fp8", "fp4x2"])
def test_dtype_main_dispatch(dtype, h):
    """The main workload with a one-byte payload, at full size: dispatch
    bit-exact against the oracle."""
    wl = workload("main").replace(dtype=dtype, h=h)
    inputs = make_inputs(wl)
    ref = oracle.dispatch(wl.cfg(), inputs["x"], inputs["topk_idx"], inputs["topk_w"])
    with DeviceRun(wl.cfg(), inputs) as run:
        run.dispatch()
        torch.cuda.synchronize()
        compare_dispatch(run, ref)
        assert run.error_word() == 0


def _check_scaled(cfg, inputs, sw, seed=7):
    rng = np.random.default_rng(seed)
    W, T = cfg["worldSize"], cfg["maxTokPerRank"]
    scales = rng.standard_normal((W, T, sw)).astype(np.float32)
    ref = oracle.dispatch(cfg, inputs["x"], inputs["topk_idx"], inputs.get("topk_w"), scales=scales)
    with DeviceRun(cfg, inputs) as run:
        R = run.info.maxRecv
        rs = torch.full((W, R, sw), 0x0C0FFEE, dtype=torch.int32, device="cuda")
        ep.ep_dispatch_scaled(run.plan, run.x, run.idx, run.w, to_dev(scales), sw, run.recv_x,
                              run.recv_meta, rs, run.recv_count, torch.cuda.current_stream())
        torch.cuda.synchronize()
        compare_dispatch(run, ref)
        ref_s = torch.from_numpy(ref["recv_scales"].view(np.int32)).to("cuda")
        for pe in range(W):
            n = int(ref["recv_count"][pe])
            assert torch.equal(rs[pe, :n], ref_s[pe, :n]), f"scale rows differ at pe {pe}"
            assert bool((rs[pe, n:] == 0x0C0FFEE).all()), f"scale rows written past count at pe {pe}"
        assert run.error_word() == 0


@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
@pytest.mark.parametrize("dtype,h,sw", [(2, 7168, 56), (0, 1024, 1), (3, 512, 33)],
                         ids=["fp8-block-scales", "bf16-one-scale", "fp4x2-33-words"])
def test_dispatch_scaled(dtype, h, sw, fused, monkeypatch):
    """Per-token scale rows travel with the payload to every destination."""
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    wl = workload("pr599").replace(dtype=dtype, h=h)
    _check_scaled(wl.cfg(), make_inputs(wl), sw)


@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
def test_dispatch_scaled_random_small(fused, monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    rng = np.random.default_rng(31)
    for case in range(6):
        cfg, xb, idx, w = P.random_small_case(rng, dtype=case % 4)
        _check_scaled(cfg, dict(x=xb, topk_idx=idx, topk_w=w), int(rng.integers(1, 80)), seed=case)


@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
def test_out_of_range_ids_reported_and_masked(fused, monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    rng = np.random.default_rng(5)
    cfg, inputs = _small_random_cfg(rng, 4, 64, 64, 4, 4, True, oob=True)
    assert (inputs["topk_idx"] >= 16).any()
    run, ref = run_and_compare(cfg, inputs)  # checks the error word against the oracle status
    assert ref["status"] == oracle.STATUS_EXPERT_RANGE
    run.close()


def test_fma_single_rounding_case():
    """The crafted input where fusing w*y into the add decides the bf16 result."""
    cfg, idx, w, y = P.fma_sensitive_case()
    inputs = dict(x=np.zeros((2, 1, 8), np.uint16), topk_idx=idx, topk_w=w)
    run, _ = run_and_compare(cfg, inputs, y_override=y)
    assert bool((run.out[0, 0] == 0x3F81).all())
    run.close()


@pytest.mark.parametrize("fused", ["0", "1"], ids=["split", "fused"])
def test_absent_tokens_and_empty_call(fused, monkeypatch):
    """All ids masked: nothing received, zero counts, zero output rows."""
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    wl = workload("latency1")
    inputs = make_inputs(wl)
    inputs["topk_idx"][:] = -1
    run, ref = run_and_compare(wl.cfg(), inputs)
    assert int(ref["recv_count"].sum()) == 0
    assert bool((run.out == 0).all())
    run.close()


def test_repeated_calls_and_reset():
    """Two dispatches with different routing on one plan: counters and the
    tile ticket reset, results follow each call."""
    wl = workload("pr599").replace(h=512)
    cfg = wl.cfg()
    a = make_inputs(wl)
    b = make_inputs(wl.replace(seed=77))
    ref_a = oracle.dispatch(cfg, a["x"], a["topk_idx"], a["topk_w"])
    ref_b = oracle.dispatch(cfg, b["x"], b["topk_idx"], b["topk_w"])
    with DeviceRun(cfg, a) as run:
        run.dispatch()
        torch.cuda.synchronize()
        compare_dispatch(run, ref_a)
        run.load_inputs(b)
        run.reset_canaries()
        run.dispatch()
        run.combine()
        torch.cuda.synchronize()
        compare_dispatch(run, ref_b)
        compare_combine(run, oracle.combine(cfg, ref_b["recv_x"], ref_b["slotmap"], ref_b["wsum"]))
        assert run.error_word() == 0


def test_combine_repeated_on_one_routing():
    """Several combines after one dispatch (e.g. for several expert outputs):
    each follows the same routing; the token counter resets between calls."""
    wl = workload("pr599").replace(h=1024)
    cfg = wl.cfg()
    inputs = make_inputs(wl)
    run, ref = run_and_compare(cfg, inputs)
    rng = np.random.default_rng(3)
    for _ in range(3):
        y = rng.integers(0, 1 << 16, size=(wl.W, wl.max_recv, wl.h)).astype(np.uint16)
        y = np.where((y & 0x7F80) == 0x7F80, y & 0x807F, y).astype(np.uint16)
        run.combine(y=to_dev(y.view(np.int16)))
        torch.cuda.synchronize()
        compare_combine(run, oracle.combine(cfg, y, ref["slotmap"], ref["wsum"]))
    assert run.error_word() == 0
    run.close()


def test_graph_capture_replay():
    """dispatch -> identity expert -> combine captured as one CUDA graph and
    replayed: every replay reproduces eager bit for bit (MORI JIT v2 design
    page §4: the graph-capture test)."""
    wl = workload("pr599")
    cfg = wl.cfg()
    inputs = make_inputs(wl)
    run, ref = run_and_compare(cfg, inputs)  # eager pass, checked against the oracle
    eager_out = run.out.clone()
    eager_meta = run.recv_meta.clone()
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
        assert torch.equal(run.recv_meta, eager_meta)
        assert np.array_equal(run.recv_count.cpu().numpy(), ref["recv_count"])
    assert run.error_word() == 0
    del g
    run.close()


@pytest.mark.parametrize("env", [
    {"EP_SCATTER_STAGES": "2"},
    {"EP_SCATTER_STAGES": "4", "EP_SCATTER_CHUNK": "4096"},  # rows in pieces, a short ring
    {"EP_SCATTER_WARPS": "1", "EP_SCATTER_BLOCKS": "1"},   # one copy engine does everything
    {"EP_SCATTER_WARPS": "16", "EP_SCATTER_STAGES": "2", "EP_SCATTER_CHUNK": "1024"},
    {"EP_COMBINE_WARPS": "1", "EP_COMBINE_BLOCKS": "3"},
    {"EP_DISPATCH_FUSED": "0"},                              # two launches: route_count + scatter_rows
    {"EP_DISPATCH_FUSED": "1", "EP_SCATTER_BLOCKS": "40"},   # fused, 52 tokens a block
    {"EP_DISPATCH_FUSED": "1", "EP_SCATTER_WARPS": "8", "EP_SCATTER_STAGES": "2", "EP_SCATTER_CHUNK": "1024"},
    {"EP_DISPATCH_FUSED": "1", "EP_SCATTER_WARPS": "1"},    # fused, one engine a block
    {"EP_SCATTER_SCAN": "route"},                            # route_count's last block scans the counts
    {"EP_DISPATCH_DENSE": "1"},                              # route_count's large-batch form
    {"EP_DISPATCH_FUSED": "1", "EP_SCATTER_BLOCKS": "7"},    # 293 tokens a block: over the bound, split
])
def test_geometry_overrides(env, monkeypatch):
    for k_, v in env.items():
        monkeypatch.setenv(k_, v)
    wl = workload("pr599").replace(h=1536)
    run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
    info = run.info
    if "EP_SCATTER_BLOCKS" in env:
        assert info.scatterBlocks == int(env["EP_SCATTER_BLOCKS"])
    if "EP_DISPATCH_FUSED" in env:
        assert info.dispatchFused == _fused_expected(info, env["EP_DISPATCH_FUSED"], wl.W * wl.max_tok)
    run.close()


def test_host_side_rejections():
    wl = workload("tiny")
    with DeviceRun(wl.cfg(), make_inputs(wl)) as run:
        with pytest.raises(ep.EpError) as e:
            run.combine()
        assert e.value.code == ep.EP_ERR_STATE
        with pytest.raises(ep.EpError) as e:
            ep.ep_dispatch(run.plan, run.x.data_ptr() + 2, run.idx, run.w, run.recv_x, run.recv_meta,
                           run.recv_count, torch.cuda.current_stream())
        assert e.value.code == ep.EP_ERR_ALIGN
        with pytest.raises(ep.EpError) as e:
            ep.ep_dispatch(run.plan, run.x, run.idx, None, run.recv_x, run.recv_meta, run.recv_count,
                           torch.cuda.current_stream())
        assert e.value.code == ep.EP_ERR_INVALID
        assert run.error_word() == 0


def test_all_workloads_registered():
    assert {"tiny", "pr599", "main", "latency1", "latency8", "skewed"} <= set(WORKLOADS)
