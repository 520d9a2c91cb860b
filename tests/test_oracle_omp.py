"""The OpenMP build of the oracle (the same C source, used to time the oracle
on all host cores) against the single-threaded build: every pin passes on it,
and both give the same bytes on the same inputs, since every output element is
computed by the same steps in the same order."""
import numpy as np
import pytest

import oracle
import oracle_pins as P
from synth.inputs import make_inputs, workload


@pytest.fixture(scope="module")
def omp():
    lib = oracle.load_omp()
    if oracle.threads(lib) < 2:
        pytest.skip("one host core: the OpenMP build would run single-threaded")
    return lib


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pins_pass_on_openmp_build(omp, pin):
    pin(lib=omp)


def _both(cfg, inputs, lib):
    r = oracle.dispatch(cfg, inputs["x"], inputs["topk_idx"], inputs["topk_w"], lib=lib)
    y = r["recv_x"]
    if int(cfg["dtype"]) in (2, 3):  # byte payloads: a bf16 expert output of the combine leg's width
        rng = np.random.default_rng(3)
        y = rng.integers(0, 1 << 16, size=(cfg["worldSize"], oracle.recv_capacity(cfg),
                                            oracle.combine_hidden(cfg)), dtype=np.uint16)
        y &= np.uint16(0x7F7F)  # finite values
    out = oracle.combine(cfg, y, r["slotmap"], r["wsum"], lib=lib)
    return r, out


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("latency8", {}),
    ("pr599", dict(h=512)),
    ("skewed", dict(h=64, max_tok=512, ct=512, max_recv=4096)),
    ("main", dict(h=32, max_tok=256, ct=200, max_recv=2048, dtype=1)),
    ("main", dict(h=32, max_tok=256, ct=256, max_recv=2048, dtype=2)),
])
def test_openmp_build_gives_identical_results(omp, name, kw):
    wl = workload(name).replace(**kw)
    cfg, inputs = wl.cfg(), make_inputs(wl)
    a, out_a = _both(cfg, inputs, None)
    b, out_b = _both(cfg, inputs, omp)
    for key in ("recv_x", "recv_meta", "recv_count", "slotmap", "wsum"):
        assert np.array_equal(a[key].view(np.uint8), b[key].view(np.uint8)), key
    assert a["status"] == b["status"]
    assert np.array_equal(out_a.view(np.uint8), out_b.view(np.uint8))
