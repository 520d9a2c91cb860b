"""Run the CUDA path through the C ABI on torch-owned device buffers and
compare it with the CPU oracle. Used by the gpu-marked tests and by the smoke
check.

Dispatch buffers are held as raw bytes (any payload dtype); the combine leg's
buffers are bf16 bits (int16) or float32, as the plan's dtype decides.
"""
from __future__ import annotations

import numpy as np
import torch

import combine_ep_dispatch_05_b200 as ep
import oracle

CANARY_BYTE = 0xAB         # byte written into recv_x before a dispatch
CANARY_META = 0x5EADBEEF   # int32 written into recv_meta before a dispatch
CANARY_OUT = 0x7FC1        # bf16 NaN bits written into out before a combine


def to_dev(a, dtype=None):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    t = torch.from_numpy(a)
    if dtype is not None:
        t = t.view(dtype)
    return t.to("cuda", non_blocking=False)


def as_bytes(a: np.ndarray) -> np.ndarray:
    """The bytes of a numpy array, as uint8 with the last axis in bytes."""
    a = np.ascontiguousarray(a)
    return a.view(np.uint8).reshape(a.shape[:-1] + (-1,))


def combine_torch_dtype(cfg):
    return torch.float32 if int(cfg["dtype"]) == 1 else torch.int16


def random_combine_input(cfg, seed=12345):
    """A seeded expert output in the combine leg's type and shape (used when the
    combine cannot take the dispatched rows as they are: fp8 / fp4x2 plans)."""
    rng = np.random.default_rng(seed)
    W, R, hc = int(cfg["worldSize"]), oracle.recv_capacity(cfg), oracle.combine_hidden(cfg)
    vals = rng.standard_normal((W, R, hc), dtype=np.float32)
    if int(cfg["dtype"]) == 1:
        return vals
    import oracle_pins
    return oracle_pins.torch_bf16_bits(vals)


class DeviceRun:
    """One plan plus the device buffers of one workload."""

    def __init__(self, cfg: dict, inputs: dict):
        self.cfg = dict(cfg)
        self.plan = ep.ep_plan_create(self.cfg)
        self.info = ep.ep_plan_info(self.plan)
        W, T, k = cfg["worldSize"], cfg["maxTokPerRank"], cfg["numExpertPerToken"]
        R, row = self.info.maxRecv, self.info.rowBytes
        hc = self.info.combineHidden
        self.shape = (W, T, k, R, row, hc)
        self.x = to_dev(as_bytes(inputs["x"]))
        assert tuple(self.x.shape) == (W, T, row)
        self.idx = to_dev(inputs["topk_idx"])
        self.w = None if inputs.get("topk_w") is None else to_dev(inputs["topk_w"])
        self.recv_x = torch.empty((W, R, row), dtype=torch.uint8, device="cuda")
        self.recv_meta = torch.empty((W, R, 3 + k), dtype=torch.int32, device="cuda")
        self.recv_count = torch.empty((W,), dtype=torch.int32, device="cuda")
        self.out = torch.empty((W, T, hc), dtype=combine_torch_dtype(cfg), device="cuda")
        self.reset_canaries()

    def reset_canaries(self):
        self.recv_x.fill_(CANARY_BYTE)
        self.recv_meta.fill_(CANARY_META)
        self.recv_count.fill_(-7)
        self.out.view(torch.int16).fill_(CANARY_OUT)

    def load_inputs(self, inputs: dict):
        self.x.copy_(to_dev(as_bytes(inputs["x"])))
        self.idx.copy_(to_dev(inputs["topk_idx"]))
        if self.w is not None:
            self.w.copy_(to_dev(inputs["topk_w"]))

    def identity_y(self):
        """The dispatched rows as the expert output, when the combine leg has
        the payload's type (bf16 and fp32 plans)."""
        assert int(self.cfg["dtype"]) in (0, 1)
        W, T, k, R, row, hc = self.shape
        return self.recv_x.view(combine_torch_dtype(self.cfg)).view(W, R, hc)

    def dispatch(self, stream=None):
        s = stream or torch.cuda.current_stream()
        ep.ep_dispatch(self.plan, self.x, self.idx, self.w, self.recv_x, self.recv_meta,
                       self.recv_count, s)

    def combine(self, y=None, stream=None):
        s = stream or torch.cuda.current_stream()
        ep.ep_combine(self.plan, self.identity_y() if y is None else y, self.out, s)

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


def compare_dispatch(run: DeviceRun, ref: dict):
    """Bit-exact comparison of dispatch outputs, on the device. Rows and
    records past recv_count must still hold the canary."""
    W = run.shape[0]
    got_count = run.recv_count.cpu().numpy()
    assert np.array_equal(got_count, ref["recv_count"]), (got_count, ref["recv_count"])
    ref_x = as_bytes(ref["recv_x"])
    for pe in range(W):
        n = int(ref["recv_count"][pe])
        assert torch.equal(run.recv_x[pe, :n], torch.from_numpy(ref_x[pe, :n]).to("cuda")), \
            f"recv_x differs at pe {pe}"
        assert bool((run.recv_x[pe, n:] == CANARY_BYTE).all()), f"recv_x written past count at pe {pe}"
        ref_meta = torch.from_numpy(ref["recv_meta"][pe, :n]).to("cuda")
        assert torch.equal(run.recv_meta[pe, :n], ref_meta), f"recv_meta differs at pe {pe}"
        assert bool((run.recv_meta[pe, n:] == CANARY_META).all()), f"meta written past count at pe {pe}"


def compare_combine(run: DeviceRun, ref_out: np.ndarray):
    """Combine: the tolerance of the spec (|d| <= 2^-7 |oracle| + 1e-3), and
    bit-exactness, since both sides fold in the same order with one rounding
    per term. A NaN must be a NaN on both sides; its sign and payload bits
    are not compared (the library leaves them unspecified: the device's fma
    and conversion give the canonical NaN, the C oracle keeps payloads)."""
    got = run.out
    if got.dtype == torch.float32:
        ref = torch.from_numpy(np.ascontiguousarray(ref_out, dtype=np.float32)).to("cuda")
        gf, rf = got, ref
        got_bits, ref_bits = got.view(torch.int32), ref.view(torch.int32)
    else:
        ref = torch.from_numpy(np.ascontiguousarray(ref_out).view(np.int16)).to("cuda")
        gf = got.view(torch.bfloat16).float()
        rf = ref.view(torch.bfloat16).float()
        got_bits, ref_bits = got, ref
    both_nan = torch.isnan(gf) & torch.isnan(rf)
    diff = (gf - rf).abs()
    # Equal values pass outright: inf - inf is NaN, not a difference.
    ok = (gf == rf) | (diff <= 2.0 ** -7 * rf.abs() + 1e-3) | both_nan
    assert bool(ok.all()), f"combine outside tolerance: max diff {float(diff[~ok].max())}"
    neq = (got_bits != ref_bits) & ~both_nan
    assert not bool(neq.any()), f"combine not bit-exact at {int(neq.sum())} elements"


def run_and_compare(cfg: dict, inputs: dict, y_override=None):
    """Oracle and GPU on the same inputs; returns (run, ref) after comparing.
    The combine runs on the dispatched rows (identity expert) when the plan's
    combine leg has the payload's type, else on a seeded expert output."""
    ref = oracle.dispatch(cfg, inputs["x"], inputs["topk_idx"], inputs.get("topk_w"))
    if y_override is None and int(cfg["dtype"]) in (2, 3):
        y_override = random_combine_input(cfg)
    y_np = ref["recv_x"] if y_override is None else y_override
    ref_out = oracle.combine(cfg, y_np, ref["slotmap"], ref["wsum"])
    run = DeviceRun(cfg, inputs)
    try:
        run.dispatch()
        if y_override is None:
            run.combine()
        else:
            run.combine(y=to_dev(np.ascontiguousarray(y_override)).view(combine_torch_dtype(cfg)))
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
