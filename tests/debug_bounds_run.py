"""Run in a process of its own with EP_B200_LIBRARY=debug (the bounds-checking
build, loaded by the binding at import): the parity suite's small cases must
match the oracle with a clean error word; with EP_TEST_BOUNDS_ROWS set below
the receive capacity, the checks must fire (EP_DEVERR_BOUNDS) and the rows
they stopped must stay unwritten. Prints "ok" and exits 0 on success."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path[:0] = [ROOT, os.path.join(ROOT, "tests")]

import numpy as np  # noqa: E402
import torch  # noqa: E402

import combine_ep_dispatch_05_b200 as ep  # noqa: E402
from combine_ep_dispatch_05_b200 import binding  # noqa: E402
from gpu_harness import CANARY_BYTE, DeviceRun, run_and_compare  # noqa: E402
from synth.inputs import make_inputs, workload  # noqa: E402


def main(mode: str) -> int:
    assert binding.LIB_PATH.endswith("libep_b200_debug.so"), binding.LIB_PATH
    torch.cuda.set_device(0)
    if mode == "clean":
        cases = [workload("tiny"), workload("pr599").replace(h=1024), workload("latency8"),
                 workload("tiny").replace(dtype=2, h=256), workload("tiny").replace(dtype=1, h=64),
                 workload("skewed").replace(h=256, max_tok=512, ct=512, max_recv=4096)]
        for wl in cases:
            run, _ = run_and_compare(wl.cfg(), make_inputs(wl))  # also asserts a clean error word
            run.close()
        # the same through the fused one-launch dispatch (read at plan creation)
        os.environ["EP_DISPATCH_FUSED"] = "1"
        for wl in cases[:3]:
            run, _ = run_and_compare(wl.cfg(), make_inputs(wl))
            assert run.info.dispatchFused == 1
            run.close()
        del os.environ["EP_DISPATCH_FUSED"]
        # the scaled dispatch: scale rows checked as well
        wl = workload("pr599").replace(h=512)
        inputs = make_inputs(wl)
        run = DeviceRun(wl.cfg(), inputs)
        sw = 4
        scales = torch.arange(wl.W * wl.max_tok * sw, dtype=torch.int32, device="cuda")
        rs = torch.zeros((wl.W, run.info.maxRecv, sw), dtype=torch.int32, device="cuda")
        ep.ep_dispatch_scaled(run.plan, run.x, run.idx, run.w, scales, sw, run.recv_x, run.recv_meta, rs,
                              run.recv_count, torch.cuda.current_stream())
        assert run.error_word() == 0
        run.close()
    else:
        wl = workload("pr599").replace(h=1024)
        half = wl.max_recv // 2
        os.environ["EP_TEST_BOUNDS_ROWS"] = str(half)
        for fused in ("0", "1"):  # both dispatch forms
            os.environ["EP_DISPATCH_FUSED"] = fused
            run = DeviceRun(wl.cfg(), make_inputs(wl))
            assert run.info.dispatchFused == int(fused)
            run.dispatch()
            torch.cuda.synchronize()
            err = run.error_word()
            assert err & ep.EP_DEVERR_BOUNDS, err
            counts = run.recv_count.cpu().numpy()
            assert (counts > half).any(), counts  # the case reaches past the checked rows
            for pe in range(wl.W):
                assert bool((run.recv_x[pe, half:] == CANARY_BYTE).all()), pe  # stopped rows stayed unwritten
            run.close()
        del os.environ["EP_DISPATCH_FUSED"]
    print("ok")
    return 0


if __name__ == "__main__":
    sys.exit(main(sys.argv[1]))
