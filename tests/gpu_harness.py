"""Run the CUDA path through the C ABI on torch-owned device buffers and
compare it with the CPU oracle. Used by the gpu-marked tests and by the smoke
check."""
from __future__ import annotations

import numpy as np
import torch

import combine_ep_dispatch_05_b200 as ep
import oracle

CANARY_X = 0xABCD          # bf16 bits written into recv_x before a dispatch
CANARY_META = 0x5EADBEEF   # int32 written into recv_meta before a dispatch


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to("cuda", non_blocking=False)


def u16(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16)


class GpuRun:
    """One plan plus the device buffers of one workload."""

    def __init__(self, cfg: dict, inputs: dict):
        self.cfg = dict(cfg)
        self.plan = ep.ep_plan_create(self.cfg)
        self.info = ep.ep_plan_info(self.plan)
        W, T, h, k = cfg["worldSize"], cfg["maxTokPerRank"], cfg["hiddenDim"], cfg["numExpertPerToken"]
        R = self.info.maxRecv
        self.shape = (W, T, h, k, R)
        self.x = to_dev(inputs["x"].view(np.int16))
        self.idx = to_dev(inputs["topk_idx"])
        self.w = None if inputs.get("topk_w") is None else to_dev(inputs["topk_w"])
        self.recv_x = torch.full((W, R, h), CANARY_X - (1 << 16), dtype=torch.int16, device="cuda")
        self.recv_meta = torch.full((W, R, 3 + k), CANARY_META, dtype=torch.int32, device="cuda")
        self.recv_count = torch.full((W,), -7, dtype=torch.int32, device="cuda")
        self.out = torch.full((W, T, h), 0x7FC1, dtype=torch.int16, device="cuda")

    def dispatch(self, stream=None):
        s = stream or torch.cuda.current_stream()
        ep.ep_dispatch(self.plan, self.x, self.idx, self.w, self.recv_x, self.recv_meta,
                       self.recv_count, s)

    def combine(self, y=None, stream=None):
        s = stream or torch.cuda.current_stream()
        ep.ep_combine(self.plan, self.recv_x if y is None else y, self.out, s)

    def error_word(self) -> int:
        return ep.ep_plan_check_error(self.plan)

    def close(self):
        if self.plan:
            torch.cuda.synchronize()
            ep.ep_plan_destroy(self.plan)
            self.plan = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()


def compare_dispatch(run: GpuRun, ref: dict):
    """Bit-exact comparison of dispatch outputs, on the device. Rows and
    records past recv_count must still hold the canary."""
    W, T, h, k, R = run.shape
    got_count = run.recv_count.cpu().numpy()
    assert np.array_equal(got_count, ref["recv_count"]), (got_count, ref["recv_count"])
    canary_x = CANARY_X - (1 << 16)
    for pe in range(W):
        n = int(ref["recv_count"][pe])
        ref_rows = torch.from_numpy(ref["recv_x"][pe, :n].view(np.int16)).to("cuda")
        assert torch.equal(run.recv_x[pe, :n], ref_rows), f"recv_x differs at pe {pe}"
        assert bool((run.recv_x[pe, n:] == canary_x).all()), f"recv_x written past count at pe {pe}"
        ref_meta = torch.from_numpy(ref["recv_meta"][pe, :n]).to("cuda")
        assert torch.equal(run.recv_meta[pe, :n], ref_meta), f"recv_meta differs at pe {pe}"
        assert bool((run.recv_meta[pe, n:] == CANARY_META).all()), f"meta written past count at pe {pe}"


def compare_combine(run: GpuRun, ref_out: np.ndarray):
    """Combine: the tolerance of the spec (|d| <= 2^-7 |oracle| + 1e-3), and
    bit-exactness, since both sides fold in the same order with one rounding
    per term."""
    got = run.out
    ref = torch.from_numpy(ref_out.view(np.int16)).to("cuda")
    gf = got.view(torch.bfloat16).float()
    rf = ref.view(torch.bfloat16).float()
    both_nan = torch.isnan(gf) & torch.isnan(rf)
    diff = (gf - rf).abs()
    ok = (diff <= 2.0 ** -7 * rf.abs() + 1e-3) | both_nan
    assert bool(ok.all()), f"combine outside tolerance: max diff {float(diff[~ok].max())}"
    neq = (got != ref) & ~both_nan
    assert not bool(neq.any()), f"combine not bit-exact at {int(neq.sum())} elements"


def run_and_compare(cfg: dict, inputs: dict, y_override=None):
    """Oracle and GPU on the same inputs; returns (run, ref) after comparing."""
    ref = oracle.dispatch(cfg, inputs["x"], inputs["topk_idx"], inputs.get("topk_w"))
    y_np = ref["recv_x"] if y_override is None else y_override
    ref_out = oracle.combine(cfg, y_np, ref["slotmap"], ref["wsum"])
    run = GpuRun(cfg, inputs)
    try:
        run.dispatch()
        if y_override is None:
            run.combine()
        else:
            run.combine(y=to_dev(y_override.view(np.int16)))
        torch.cuda.synchronize()
        compare_dispatch(run, ref)
        compare_combine(run, ref_out)
        err = run.error_word()
        expect = ep.EP_DEVERR_EXPERT_RANGE if ref["status"] == oracle.STATUS_EXPERT_RANGE else 0
        assert err == expect, f"device error word {err}, expected {expect}"
    except BaseException:
        run.close()
        raise
    return run, ref
