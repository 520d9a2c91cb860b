"""Benchmark: one step = ep_dispatch -> identity expert (y = recv_x) ->
ep_combine over W=8 virtual EP ranks on one B200, through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload main|pr599|skewed|latency1|latency8|mid] [--no-cpu-baseline]

Prints one JSON line (rank 0). Timing: W untimed warm-up steps, then K steps,
each bracketed by CUDA events on the launching stream (dispatch and combine
separately); L2 is flushed between steps outside the events by reading a
256 MB buffer (``--flush write`` rewrites it instead; the main workload's
inputs are larger than L2 as well). Barrier +
synchronize on both sides; the reported time is the max over ranks. N > 1
runs N independent replicas, one per GPU (each GPU holds all W virtual ranks).

--impl reference times the CPU oracle (the plain C statement of the method) on
the full workload on this host: its OpenMP build on all cores is the value, and
one step of its single-threaded build is reported beside it (``cpu_baseline``).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth.inputs import make_inputs, workload  # noqa: E402

METRIC = "dispatch+combine µs and HBM GB/s (% of B200 peak) at W=8 ct=4096 h=7168 topk8"
FALLBACK_HBM_GBS = 6650.0
FLUSH_BYTES = 256 << 20
# The device code whose DRAM traffic profiles/ncu_traffic.json records; the
# launch geometry it was taken with is recorded beside it.
KERNEL_SOURCES = ["combine_ep_dispatch_05_b200/csrc/ep_kernels.cu",
                  "combine_ep_dispatch_05_b200/csrc/ep_internal.h"]
TRAFFIC_GEOMETRY = ("scatterWarps", "scatterStages", "scatterChunkBytes", "scatterBlocks", "combineWarps",
                    "combineBlocks")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="main")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp32", "fp8", "fp4x2"],
                    help="dispatch payload type (the combine leg is fp32 for fp32, bf16 otherwise); "
                         "fp4x2 halves hiddenDim, which then counts bytes of packed pairs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the hot-L2 timing of back-to-back calls in CUDA graphs")
    ap.add_argument("--flush", default="read", choices=["read", "write"],
                    help="L2 flush between timed steps: read a 256 MB buffer (leaves L2 clean) "
                         "or write it (leaves L2 full of dirty lines)")
    return ap.parse_args()


DTYPES = {"bf16": 0, "fp32": 1, "fp8": 2, "fp4x2": 3}


def get_workload(name, dtype="bf16"):
    if name == "mid":  # the main shape at 1024 tokens/rank: the small ncu case
        wl = workload("main").replace(name="mid", max_tok=1024, ct=1024, max_recv=8192)
    else:
        wl = workload(name)
    dt = DTYPES[dtype]
    if dt == 0:
        return wl
    # fp4x2: the same element count, in hiddenDim bytes of packed pairs
    return wl.replace(name=f"{wl.name}_{dtype}", dtype=dt, h=wl.h // 2 if dt == 3 else wl.h)


def payload_bytes(wl) -> int:
    return wl.h * {0: 2, 1: 4, 2: 1, 3: 1}[wl.dtype]


def combine_row_bytes(wl) -> int:
    hc = 2 * wl.h if wl.dtype == 3 else wl.h
    return hc * (4 if wl.dtype == 1 else 2)


def describe(wl) -> dict:
    return {"workload": f"{wl.name}: W={wl.W} ct={wl.ct} h={wl.h} topk={wl.k} "
                        f"E={wl.E} ({wl.n_epr}/rank) {wl.routing} routing, bf16 rows",
            "world_size": wl.W, "tokens_per_rank": wl.ct, "max_tok_per_rank": wl.max_tok,
            "hidden": wl.h, "topk": wl.k, "experts": wl.E, "max_recv": wl.max_recv,
            "use_weights": wl.use_weights,
            "payload_dtype": {0: "bf16", 1: "fp32", 2: "fp8", 3: "fp4x2"}[wl.dtype],
            "combine_dtype": "fp32" if wl.dtype == 1 else "bf16",
            "l2": "L2 flushed between steps outside the events (256 MB buffer, see flush); "
                  "inputs larger than L2"}


def dispatch_bytes(wl, U, n_routed):
    row, G, k, W = payload_bytes(wl), wl.W * wl.max_tok, wl.k, wl.W
    return (n_routed * row                    # read each routed x row once
            + U * row                         # write every received row
            + G * k * 4 * (1 + int(wl.use_weights))  # topk ids (+ weights)
            + U * (3 + k) * 4                 # meta records
            + 4 * W)                          # recv_count


def combine_bytes(wl, U):
    row, G = combine_row_bytes(wl), wl.W * wl.max_tok
    return (U * row       # read every received row of y
            + G * row     # write every out row
            + U * 8)      # (slot, weight) of each received row


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_hash() -> str:
    """Hash of the kernel sources' code: comments and whitespace are left out,
    so that a recorded traffic figure survives edits that change no code."""
    import re
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, wl_name: str, geometry: dict):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel code with the launch geometry this run has; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel]
        if e.get("source_sha") != source_hash():
            return None
        rec = d["geometry"][wl_name]
        if any(rec[k] != geometry.get(k) for k in TRAFFIC_GEOMETRY):
            return None
        return e["per_launch_bytes"].get(wl_name)
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.t0 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        self.t0 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        # samples under load: the top 3/4 of power draw
        cut = sorted(power)[len(power) // 4] if len(power) >= 4 else min(power)
        loaded = [s for s, p in zip(sm, power) if p >= cut] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power), "reasons": sorted(reasons)}


def dist_setup(n):
    if n <= 1 and "RANK" not in os.environ:
        return 0, 1, 0, None
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    return rank, world, local, dist


def max_over_ranks(val: float, dist, device) -> float:
    if dist is None:
        return val
    import torch
    t = torch.tensor([val], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ reference arm
def host_cpu() -> dict:
    """The host's usable cores and its CPU model."""
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except Exception:
        pass
    return {"nproc": cores, "cpu_model": model}


def time_oracle(wl, inputs, steps, lib=None):
    """Seconds of (dispatch, combine) per oracle step on the full workload.
    lib: an oracle build (None: the single-threaded one). The receive and
    output buffers are allocated once, outside the timed calls."""
    import oracle
    cfg = wl.cfg()
    R = oracle.recv_capacity(cfg)
    recv_x = np.zeros((wl.W, R, wl.h), dtype=oracle.payload_np(cfg))
    recv_meta = np.zeros((wl.W, R, 3 + wl.k), dtype=np.int32)
    out = np.zeros((wl.W, wl.max_tok, oracle.combine_hidden(cfg)), dtype=oracle.combine_np(cfg))
    idx = inputs["topk_idx"]
    y = None
    if wl.dtype in (2, 3):  # one-byte payloads: the expert hands back bf16 rows
        rng = np.random.default_rng(wl.seed)
        y = rng.integers(0x3C00, 0x4000, size=(wl.W, R, oracle.combine_hidden(cfg)), dtype=np.uint16)
        y |= (rng.integers(0, 2, size=y.shape, dtype=np.uint16) << 15)
    ts = []
    for _ in range(steps):
        t0 = time.perf_counter()
        r = oracle.dispatch(cfg, inputs["x"], idx, inputs["topk_w"], recv_x=recv_x, recv_meta=recv_meta,
                            lib=lib)
        t1 = time.perf_counter()
        oracle.combine(cfg, r["recv_x"] if y is None else y, r["slotmap"], r["wsum"], lib=lib, out=out)
        ts.append((t1 - t0, time.perf_counter() - t1))
    return ts


def cpu_baseline(wl, inputs, steps, warmup, single_steps=1) -> dict:
    """The oracle on this host: the OpenMP build on all cores (the value),
    and the single-threaded build for one step beside it. Both run the full
    workload; their results are identical."""
    import oracle
    oracle.build()
    omp = oracle.load_omp()
    threads = oracle.threads(omp)
    time_oracle(wl, inputs, warmup, omp)
    ts = time_oracle(wl, inputs, steps, omp)
    one = time_oracle(wl, inputs, single_steps, None)
    mean = lambda xs: statistics.mean(xs) * 1e6  # noqa: E731
    return {"value": mean([d + c for d, c in ts]), "unit": "us", "cores": threads, "kind": "oracle",
            "sample": (f"the full {wl.name} workload, {steps} steps after {warmup} warm-up, OpenMP build of "
                       f"the C oracle on {threads} threads (dispatch shares out the {wl.W} destinations, "
                       f"combine the tokens); single-threaded build for {single_steps} step(s) beside it"),
            "dispatch_us": mean([d for d, _ in ts]), "combine_us": mean([c for _, c in ts]),
            "single_core_us": mean([d + c for d, c in one]),
            "single_core_dispatch_us": mean([d for d, _ in one]),
            "single_core_combine_us": mean([c for _, c in one]), **host_cpu()}


def run_reference(args, wl):
    rank, world, local, dist = dist_setup(args.gpus)
    if rank != 0:
        return 0
    if world > 1:  # the arm's config: the same workload with its W ranks on the N GPUs
        wl = comm_workload(wl, world)
    inputs = make_inputs(wl)
    cpu = cpu_baseline(wl, inputs, args.steps, args.warmup)
    us = cpu["value"]
    line = {"metric": METRIC, "value": us, "unit": "us", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": us / 1e3, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None,
            "dtype": {0: "bf16", 1: "f32", 2: "fp8", 3: "fp4x2"}[wl.dtype], "data": "synthetic",
            "config": describe(wl), "impl": "reference", "cpu_baseline": cpu,
            "e2e": {"value": us, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def dispatch_kernels(info) -> str:
    """The kernels one dispatch of this plan launches."""
    if info.dispatchFused:
        return "ep_dispatch_fused (one launch)"
    return "ep_dispatch (route_count + scatter_rows)"


def dispatch_launches(info) -> int:
    return 1 if info.dispatchFused else 2


GRAPH_CALLS = 20   # calls captured back to back in one CUDA graph
GRAPH_ROUNDS = 10  # timed replays of each graph, interleaved


def time_graphs(calls: dict, dev, dist) -> dict:
    """Hot-L2 device time per call. Each entry of ``calls`` (a function of the
    stream) is captured GRAPH_CALLS times back to back in one CUDA graph. The
    graphs are replayed in turn, GRAPH_ROUNDS timed rounds after two untimed
    ones, each replay bracketed by CUDA events on its stream; the result is the
    median replay ÷ GRAPH_CALLS (max over ranks). Launch overhead is left out
    and consecutive calls may overlap through programmatic dependent launch,
    so this is the per-call cost of a steady stream of calls."""
    import torch
    cs = torch.cuda.Stream(dev)
    cs.wait_stream(torch.cuda.current_stream(dev))
    graphs = {}
    for name, fn in calls.items():
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                for _ in range(GRAPH_CALLS):
                    fn(cs)
        graphs[name] = g
    times = {name: [] for name in graphs}
    with torch.cuda.stream(cs):
        for r in range(GRAPH_ROUNDS + 2):
            for name, g in graphs.items():
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(cs)
                g.replay()
                e1.record(cs)
                if r >= 2:
                    times[name].append((e0, e1))
    torch.cuda.synchronize(dev)
    res = {}
    for name, evs in times.items():
        med = statistics.median(a.elapsed_time(b) for a, b in evs) / GRAPH_CALLS
        res[name + "_us"] = max_over_ranks(med, dist, dev) * 1e3
    for g in graphs.values():
        del g
    graphs.clear()
    res.update({"calls_per_graph": GRAPH_CALLS, "rounds": GRAPH_ROUNDS, "l2": "hot (no flush)",
                "statistic": "median replay / calls"})
    return res


def run_ours(args, wl):
    import torch
    rank, world, local, dist = dist_setup(args.gpus)
    # EP_BENCH_COMM=1 (under torchrun) runs the communicator path with one rank
    # as well: the device-barrier path of a multi-GPU run, on one GPU.
    if world > 1 or (dist is not None and os.environ.get("EP_BENCH_COMM") == "1"):
        return run_comm(args, wl, rank, world, local, dist)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist is not None:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    from combine_ep_dispatch_05_b200 import build as epbuild
    if rank == 0 or dist is None:
        epbuild.build()
    if dist is not None:
        dist.barrier()
    import combine_ep_dispatch_05_b200 as ep

    cfg = wl.cfg()
    inputs = make_inputs(wl)
    plan = ep.ep_plan_create(cfg)
    info = ep.ep_plan_info(plan)
    W, T, h, k, R = wl.W, wl.max_tok, wl.h, wl.k, info.maxRecv
    x = torch.from_numpy(inputs["x"].view(np.uint8).reshape(W, T, -1)).to(dev)
    idx = torch.from_numpy(inputs["topk_idx"]).to(dev)
    w = torch.from_numpy(inputs["topk_w"]).to(dev) if inputs["topk_w"] is not None else None
    recv_x = torch.empty((W, R, info.rowBytes), dtype=torch.uint8, device=dev)
    recv_meta = torch.empty((W, R, 3 + k), dtype=torch.int32, device=dev)
    recv_count = torch.empty((W,), dtype=torch.int32, device=dev)
    cdt = torch.float32 if wl.dtype == 1 else torch.bfloat16
    out = torch.empty((W, T, info.combineHidden), dtype=cdt, device=dev)
    if wl.dtype in (0, 1):
        y = recv_x.view(cdt).view(W, R, info.combineHidden)  # identity expert: y = recv_x
    else:
        # one-byte payloads: the expert hands back bf16 rows (seeded, made on the device)
        gen = torch.Generator(device=dev)
        gen.manual_seed(wl.seed)
        y = torch.randn((W, R, info.combineHidden), generator=gen, device=dev).to(cdt)
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_out = torch.empty(1, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)

    def flush_l2(i):
        if args.flush == "write":
            flush.fill_(i)
        else:  # read it: evicts L2 and leaves only clean lines behind
            torch.amax(flush, dim=0, out=flush_out.view(()))

    def step():
        ep.ep_dispatch(plan, x, idx, w, recv_x, recv_meta, recv_count, s)
        ep.ep_combine(plan, y, out, s)

    for i in range(max(args.warmup, 0)):
        flush_l2(i)
        step()
    torch.cuda.synchronize(dev)
    err = ep.ep_plan_check_error(plan)
    if err:
        raise RuntimeError(f"device error word {err} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    t_wall = time.perf_counter()
    for i in range(args.steps):
        flush_l2(i + 1)
        evs[i][0].record(s)
        ep.ep_dispatch(plan, x, idx, w, recv_x, recv_meta, recv_count, s)
        evs[i][1].record(s)
        ep.ep_combine(plan, y, out, s)
        evs[i][2].record(s)
    torch.cuda.synchronize(dev)
    t_wall = time.perf_counter() - t_wall
    if dist is not None:
        dist.barrier()
    clocks = sampler.stop()
    t_disp = [evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps)]
    t_comb = [evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps)]
    disp_ms = statistics.mean(t_disp)
    comb_ms = statistics.mean(t_comb)
    step_ms = max_over_ranks(disp_ms + comb_ms, dist, dev)
    disp_ms_max = max_over_ranks(disp_ms, dist, dev)
    comb_ms_max = max_over_ranks(comb_ms, dist, dev)
    err = ep.ep_plan_check_error(plan)
    if err:
        raise RuntimeError(f"device error word {err} after the timed steps")

    graph = None
    if not args.no_graph:
        graph = time_graphs({
            "dispatch": lambda st: ep.ep_dispatch(plan, x, idx, w, recv_x, recv_meta, recv_count, st),
            "combine": lambda st: ep.ep_combine(plan, y, out, st),
            "pair": lambda st: (ep.ep_dispatch(plan, x, idx, w, recv_x, recv_meta, recv_count, st),
                                ep.ep_combine(plan, y, out, st)),
        }, dev, dist)
        err = ep.ep_plan_check_error(plan)
        if err:
            raise RuntimeError(f"device error word {err} after the graph timing")

    # Algorithmic bytes from the actual routing.
    counts = recv_count.cpu().numpy()
    U = int(counts.sum())
    n_routed = int((inputs["topk_idx"] >= 0).any(axis=-1).sum())
    db, cb = dispatch_bytes(wl, U, n_routed), combine_bytes(wl, U)
    peak, peak_src = hbm_peak()
    d_gbs = db / (disp_ms_max * 1e-3) / 1e9
    c_gbs = cb / (comb_ms_max * 1e-3) / 1e9
    pair_gbs = (db + cb) / (step_ms * 1e-3) / 1e9
    if comb_ms_max >= disp_ms_max:
        dom = {"kernel": "ep_combine_kernel", "bytes": cb, "ms": comb_ms_max, "gbs": c_gbs}
    else:
        dom = {"kernel": dispatch_kernels(info), "bytes": db, "ms": disp_ms_max, "gbs": d_gbs}
    traffic = ncu_traffic("ep_combine_kernel" if dom["kernel"] == "ep_combine_kernel" else "ep_dispatch", wl.name,
                          info.as_dict())

    # End to end: every step copies its inputs from pinned host memory to the
    # device, runs dispatch and combine, and copies its result back to pinned
    # host memory. Steps are double-buffered on three streams (host->device,
    # compute, device->host) so that one step's upload overlaps the previous
    # step's download, as a serving loop would run them.
    e2e = None
    if not args.no_e2e:
        x_h = torch.from_numpy(inputs["x"].view(np.uint8).reshape(W, T, -1)).pin_memory()
        idx_h = torch.from_numpy(inputs["topk_idx"]).pin_memory()
        w_h = torch.from_numpy(inputs["topk_w"]).pin_memory() if w is not None else None
        out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        xs, idxs, ws = [x, torch.empty_like(x)], [idx, torch.empty_like(idx)], [w, None if w is None else torch.empty_like(w)]
        outs = [out, torch.empty_like(out)]
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_free = [torch.cuda.Event() for _ in range(2)]    # compute finished with input set b
        in_ready = [torch.cuda.Event() for _ in range(2)]   # upload of input set b finished
        out_ready = [torch.cuda.Event() for _ in range(2)]  # combine wrote out set b
        out_free = [torch.cuda.Event() for _ in range(2)]   # download of out set b finished
        for b in range(2):
            in_free[b].record(s)
            out_free[b].record(s)

        def e2e_step(i):
            b = i & 1
            with torch.cuda.stream(s_up):
                s_up.wait_event(in_free[b])
                xs[b].copy_(x_h, non_blocking=True)
                idxs[b].copy_(idx_h, non_blocking=True)
                if w_h is not None:
                    ws[b].copy_(w_h, non_blocking=True)
                in_ready[b].record(s_up)
            s.wait_event(in_ready[b])
            ep.ep_dispatch(plan, xs[b], idxs[b], ws[b], recv_x, recv_meta, recv_count, s)
            in_free[b].record(s)
            s.wait_event(out_free[b])
            ep.ep_combine(plan, y, outs[b], s)
            out_ready[b].record(s)
            with torch.cuda.stream(s_down):
                s_down.wait_event(out_ready[b])
                out_h[b].copy_(outs[b], non_blocking=True)
                out_free[b].record(s_down)

        for i in range(max(1, min(args.warmup, 3))):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        # Enough steps that the pipeline's fill (the first upload alone) and
        # drain (the last download alone) weigh little against the steady state.
        n_e2e = max(2, min(args.steps, 50))
        e0.record(s_up)
        for i in range(n_e2e):
            e2e_step(i)
        e1.record(s_down)  # after the last download, which follows everything else
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, dev)
        # the result of the last step is the device result, byte for byte
        assert torch.equal(out_h[(n_e2e - 1) & 1], outs[(n_e2e - 1) & 1].cpu())
        h2d = x_h.numel() + idx_h.numel() * 4 + (w_h.numel() * 4 if w_h is not None else 0)
        e2e = {"value": e2e_ms * 1e3, "unit": "us", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(out_h[0].numel() * out_h[0].element_size()), "steps": n_e2e,
               "pipeline": "double-buffered: upload of step i overlaps download of step i-1"}

    ep.ep_plan_destroy(plan)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, inputs, steps=3, warmup=1)

    if rank == 0:
        line = {
            "metric": METRIC, "value": step_ms * 1e3, "unit": "us", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": {0: "bf16", 1: "f32", 2: "fp8", 3: "fp4x2"}[wl.dtype],
            "data": "synthetic",
            "config": {**describe(wl), "flush": args.flush,
                       "parallelism": "virtual EP ranks on each GPU; replicas across GPUs"},
            "dispatch_us": disp_ms_max * 1e3, "combine_us": comb_ms_max * 1e3,
            "dispatch_gbs": d_gbs, "combine_gbs": c_gbs, "pair_gbs": pair_gbs,
            "pair_frac_of_peak": pair_gbs / peak, "recv_rows_U": U,
            "algorithmic_bytes": {"dispatch": db, "combine": cb},
            "roofline": {"bound": "hbm", "kernel": dom["kernel"], "achieved": dom["gbs"], "peak": peak,
                         "peak_source": f"{peak_src} copy bandwidth", "unit": "GB/s",
                         "frac": dom["gbs"] / peak, "traffic": traffic,
                         "bytes_per_launch": dom["bytes"], "avg_launch_us": dom["ms"] * 1e3},
            "roofline_all": {
                "dispatch": {"achieved": d_gbs, "frac": d_gbs / peak, "bytes": db, "us": disp_ms_max * 1e3},
                "combine": {"achieved": c_gbs, "frac": c_gbs / peak, "bytes": cb, "us": comb_ms_max * 1e3}},
            "graph_hot": graph,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": (dispatch_launches(info) + 1) * args.steps, "timed_wall_s": t_wall,
            "geometry": info.as_dict(), "impl": "ours",
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ ranks on separate GPUs
NVLINK_PEER_GBS = 770.0  # measured peer copy per direction per GPU on this machine's B200s


def comm_workload(wl, world: int):
    """The workload with its W ranks real, one per GPU: every rank holds
    wl.max_tok token rows (wl.ct live), the experts are shared out over the
    ranks (same total E), and every rank can receive the worst case."""
    if wl.E % world:
        raise SystemExit(f"{wl.E} experts do not divide over {world} ranks")
    return wl.replace(W=world, n_epr=wl.E // world, max_recv=world * wl.max_tok)


def rank_inputs(cwl, rank: int) -> dict:
    """Rank `rank`'s seeded tokens (x, ids over all E experts, weights), made
    on that rank only."""
    one = cwl.replace(W=1, n_epr=cwl.E, max_recv=0, seed=cwl.seed * 1000 + rank)
    inp = make_inputs(one)
    return {"x": inp["x"][0], "topk_idx": inp["topk_idx"][0],
            "topk_w": None if inp["topk_w"] is None else inp["topk_w"][0]}


def nccl_alltoallv_step(x, idx, w, world: int, n_epr: int, dist):
    """The library-collective baseline of one dispatch + identity expert +
    combine: torch gathers the rows of each destination, NCCL moves them with
    all_to_all_single (sizes exchanged first, then read on the host), the
    rows go back the same way, and torch folds them (index_add in float32;
    its order is not fixed). x: uint8 [T][row bytes] of bf16 rows. Returns
    (out as bf16 [T][h], the received rows)."""
    import torch
    T, k = idx.shape
    pe = torch.where(idx >= 0, torch.div(idx, n_epr, rounding_mode="floor"), torch.full_like(idx, world))
    hit = torch.zeros((T, world + 1), dtype=torch.bool, device=x.device)
    hit.scatter_(1, pe.long(), True)
    hit = hit[:, :world]
    dest, tok = hit.t().nonzero(as_tuple=True)  # by destination, then token
    send = x.index_select(0, tok)
    send_counts = hit.sum(0).to(torch.int64)
    recv_counts = torch.empty_like(send_counts)
    dist.all_to_all_single(recv_counts, send_counts)
    sc, rc = send_counts.tolist(), recv_counts.tolist()
    recv = torch.empty((sum(rc),) + tuple(x.shape[1:]), dtype=x.dtype, device=x.device)
    dist.all_to_all_single(recv, send, rc, sc)
    back = torch.empty_like(send)
    dist.all_to_all_single(back, recv, sc, rc)  # identity expert: the rows come back
    if w is None:
        wsum = hit.to(torch.float32)
    else:
        wsum = torch.zeros((T, world + 1), dtype=torch.float32, device=x.device)
        wsum.scatter_add_(1, pe.long(), w)
        wsum = wsum[:, :world]
    rows = back.view(torch.bfloat16).float() * wsum[tok, dest].unsqueeze(1)  # rows are bytes of bf16
    out = torch.zeros((T, rows.shape[1]), dtype=torch.float32, device=x.device)
    out.index_add_(0, tok, rows)
    return out.to(torch.bfloat16), recv


def run_comm(args, wl, rank, world, local, dist):
    """N > 1: the W ranks are the N processes, one per GPU, connected by the
    library's communicator (ep_comm_*): the rows cross NVLink. Timed as the
    one-GPU step, max over ranks; the NCCL all-to-allv baseline beside it.
    EP_BENCH_SHARE_GPU=1 puts every rank on GPU 0 with host barriers and a
    gloo process group, to run this path where there is one GPU (no NCCL
    baseline then)."""
    import datetime
    import torch
    share = os.environ.get("EP_BENCH_SHARE_GPU") == "1"
    if share:
        local = 0
    dev = torch.device("cuda", local)
    torch.cuda.set_device(local)
    if share:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    else:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))
    cdev = torch.device("cpu") if share else dev  # where the bench's own collectives run
    from combine_ep_dispatch_05_b200 import build as epbuild
    if rank == 0:
        epbuild.build()
    dist.barrier()
    import combine_ep_dispatch_05_b200 as ep
    from combine_ep_dispatch_05_b200 import comm as epcomm

    cwl = comm_workload(wl, world)
    if share:
        comm = epcomm.create_and_connect(cwl.cfg(), dist, ep.EP_SYNC_HOST)
        sync = "host"
    else:
        comm = epcomm.create_and_connect(cwl.cfg(), dist, ep.EP_SYNC_DEVICE)
        sync = "device"
    info = ep.ep_comm_info(comm)
    inp = rank_inputs(cwl, rank)
    x = torch.from_numpy(inp["x"].view(np.uint8)).to(dev)
    idx = torch.from_numpy(inp["topk_idx"]).to(dev)
    w = None if inp["topk_w"] is None else torch.from_numpy(inp["topk_w"]).to(dev)
    hc = info.combineRowBytes // 2
    y = torch.as_tensor(_DeviceMemory(info.recvX, (info.maxRecv, hc), "<i2"), device=dev).view(torch.bfloat16)
    out = torch.empty((cwl.max_tok, hc), dtype=torch.bfloat16, device=dev)
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_out = torch.empty((), dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream(dev)

    for i in range(max(args.warmup, 0)):
        torch.amax(flush, dim=0, out=flush_out)
        ep.ep_comm_dispatch(comm, x, idx, w, s)
        ep.ep_comm_combine(comm, y, out, s)
    torch.cuda.synchronize(dev)
    if ep.ep_comm_check_error(comm):
        raise RuntimeError("device error word after warm-up")
    check_comm_step(cwl, inp, out, info, rank, world, dist, dev, cdev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    for i in range(args.steps):
        torch.amax(flush, dim=0, out=flush_out)
        evs[i][0].record(s)
        ep.ep_comm_dispatch(comm, x, idx, w, s)
        evs[i][1].record(s)
        ep.ep_comm_combine(comm, y, out, s)
        evs[i][2].record(s)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clocks = sampler.stop()
    disp_ms = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps))
    comb_ms = statistics.mean(evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps))
    step_ms = max_over_ranks(disp_ms + comb_ms, dist, cdev)
    disp_ms = max_over_ranks(disp_ms, dist, cdev)
    comb_ms = max_over_ranks(comb_ms, dist, cdev)
    if ep.ep_comm_check_error(comm):
        raise RuntimeError("device error word after the timed steps")

    # Rows that cross NVLink: every row a rank sends to another rank, and the
    # same rows coming back in the combine (the busiest rank sets the pace).
    recv_n = int(torch.as_tensor(_DeviceMemory(info.recvCount, (1,), "<i4"), device=dev).cpu()[0])
    T = cwl.max_tok
    ids = inp["topk_idx"]
    dest = np.where(ids >= 0, ids // cwl.n_epr, -1)
    hit = np.zeros((T, world), dtype=bool)
    for j in range(cwl.k):
        m = dest[:, j] >= 0
        hit[np.nonzero(m)[0], dest[m, j]] = True
    sent_remote = int(hit.sum() - hit[:, rank].sum())
    link_bytes = max_over_ranks(float(sent_remote * info.rowBytes), dist, cdev)
    link_gbs = link_bytes / (max(disp_ms, comb_ms) * 1e-3) / 1e9

    # The library-collective baseline on the same tokens.
    nccl = None
    if not share:
        xb = x.view(cwl.max_tok, -1)
        for _ in range(2):
            nccl_alltoallv_step(xb, idx, w, world, cwl.n_epr, dist)
        torch.cuda.synchronize(dev)
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nb = max(3, min(args.steps, 20))
        e0.record(s)
        for _ in range(nb):
            nccl_alltoallv_step(xb, idx, w, world, cwl.n_epr, dist)
        e1.record(s)
        torch.cuda.synchronize(dev)
        nccl = {"step_us": max_over_ranks(e0.elapsed_time(e1) / nb, dist, cdev) * 1e3,
                "impl": "torch gather + NCCL all_to_all_single (sizes read on the host) + torch index_add fold"}

    # End to end through the same calls: every step uploads this rank's
    # inputs from pinned host memory and downloads its output rows.
    e2e = None
    if not args.no_e2e:
        x_h = torch.from_numpy(inp["x"].view(np.uint8)).pin_memory()
        idx_h = torch.from_numpy(inp["topk_idx"]).pin_memory()
        w_h = None if w is None else torch.from_numpy(inp["topk_w"]).pin_memory()
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            x.copy_(x_h, non_blocking=True)
            idx.copy_(idx_h, non_blocking=True)
            if w_h is not None:
                w.copy_(w_h, non_blocking=True)
            ep.ep_comm_dispatch(comm, x, idx, w, s)
            ep.ep_comm_combine(comm, y, out, s)
            out_h.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        dist.barrier()
        n_e2e = max(2, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(s)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, cdev)
        h2d = x_h.numel() + idx_h.numel() * 4 + (0 if w_h is None else w_h.numel() * 4)
        e2e = {"value": e2e_ms * 1e3, "unit": "us", "h2d_bytes_per_step": int(h2d) * world,
               "d2h_bytes_per_step": int(out_h.numel() * out_h.element_size()) * world, "steps": n_e2e,
               "pipeline": "sequential on each rank; bytes are all ranks' together"}

    dist.barrier()
    ep.ep_comm_destroy(comm)
    if rank == 0:
        line = {
            "metric": METRIC, "value": step_ms * 1e3, "unit": "us", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {**describe(cwl), "flush": "read",
                       "parallelism": f"expert parallel: {world} ranks, one per GPU, rows over NVLink "
                                      f"(communicator, {sync} barriers)"},
            "dispatch_us": disp_ms * 1e3, "combine_us": comb_ms * 1e3,
            "rows_received_rank0": recv_n,
            "roofline": {"bound": "nvlink", "kernel": "ep_comm dispatch / combine",
                         "achieved": link_gbs, "peak": NVLINK_PEER_GBS,
                         "peak_source": "measured peer copy per direction per GPU (fallback figure)",
                         "unit": "GB/s", "frac": link_gbs / NVLINK_PEER_GBS, "traffic": None,
                         "bytes_per_launch": link_bytes, "avg_launch_us": max(disp_ms, comb_ms) * 1e3},
            "nccl_baseline": nccl,
            "cpu_baseline": None, "e2e": e2e, "clocks": clocks,
            "gpu_launches": 7 * args.steps, "impl": "ours",
        }
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()
    return 0


def check_comm_step(cwl, inp, out, info, rank, world, dist, dev, cdev):
    """Self-check of the last warm-up step, from this rank's own inputs: the
    rows this rank received must number what every rank's routing sends it
    (count rows gathered from all ranks), and with the identity expert every
    output row must be the row times the sum of its weight sums, within the
    spec's tolerance (float64 reference)."""
    import torch
    T, k, W = cwl.max_tok, cwl.k, world
    ids = inp["topk_idx"]
    dest = np.where(ids >= 0, ids // cwl.n_epr, -1)
    hit = np.zeros((T, W), dtype=bool)
    for j in range(k):
        m = dest[:, j] >= 0
        hit[np.nonzero(m)[0], dest[m, j]] = True
    counts = torch.from_numpy(hit.sum(0).astype(np.int64)).to(cdev)
    table = [torch.empty_like(counts) for _ in range(W)]
    dist.all_gather(table, counts)
    expect = int(sum(int(t[rank]) for t in table))
    got = int(torch.as_tensor(_DeviceMemory(info.recvCount, (1,), "<i4"), device=dev).cpu()[0])
    if got != expect:
        raise RuntimeError(f"rank {rank}: received {got} rows, the routing sends {expect}")
    xw = inp["x"].view(np.uint16).astype(np.uint32) << 16
    xf = xw.view(np.float32).astype(np.float64)
    if inp["topk_w"] is None:
        scale = hit.sum(1).astype(np.float64)
    else:
        scale = np.where(ids >= 0, inp["topk_w"], 0.0).astype(np.float64).sum(1)
    ref = xf * scale[:, None]
    o = out.float().cpu().numpy().astype(np.float64)
    bad = np.abs(o - ref) > 2.0 ** -7 * np.abs(ref) + 1e-3
    if bad.any():
        raise RuntimeError(f"rank {rank}: {int(bad.sum())} output elements outside tolerance")


class _DeviceMemory:
    """A view of library-owned device memory for torch.as_tensor."""

    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def main():
    args = parse()
    wl = get_workload(args.workload, args.dtype)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
