"""Property tests of the CPU oracle (no GPU): hypothesis draws tiny problems
(world size, tokens, topk, experts per rank, masked and duplicate ids,
weights or none, every payload type) and checks the oracle against the
brute-force set formulation of dispatch and the exact-rational fold of
combine. A failure shrinks to a smallest counterexample."""
from fractions import Fraction

import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as st  # noqa: E402

import oracle  # noqa: E402
import oracle_pins as P  # noqa: E402


@st.composite
def problems(draw):
    W = draw(st.integers(1, 5))
    T = draw(st.integers(1, 5))
    k = draw(st.integers(1, 4))
    nEpr = draw(st.integers(1, 3))
    dtype = draw(st.integers(0, 3))
    use_w = draw(st.booleans())
    E = W * nEpr
    ids = draw(st.lists(st.integers(-2, E - 1), min_size=W * T * k, max_size=W * T * k))
    idx = np.array(ids, dtype=np.int32).reshape(W, T, k)
    wts = draw(st.lists(st.floats(-4.0, 4.0, width=32, allow_subnormal=False),
                        min_size=W * T * k, max_size=W * T * k))
    w = np.array(wts, dtype=np.float32).reshape(W, T, k) if use_w else None
    h = {0: 8, 1: 4, 2: 16, 3: 16}[dtype]
    seed = draw(st.integers(0, 2 ** 32 - 1))
    xb = P.random_payload(np.random.default_rng(seed), (W, T, h), dtype)
    maxRecv = draw(st.sampled_from([0, W * T, W * T + 2]))
    cfg = dict(worldSize=W, hiddenDim=h, maxTokPerRank=T, numExpertPerRank=nEpr, numExpertPerToken=k,
               maxRecv=maxRecv, dtype=dtype, useWeights=int(use_w))
    return cfg, xb, idx, w


@settings(max_examples=80, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(problems())
def test_dispatch_matches_the_set_formulation(prob):
    cfg, xb, idx, w = prob
    W, T, k, nEpr = (cfg[n] for n in ("worldSize", "maxTokPerRank", "numExpertPerToken", "numExpertPerRank"))
    res = oracle.dispatch(cfg, xb, idx, w)
    slot, count = P.brute_routes(cfg, idx)
    assert list(res["recv_count"]) == count
    for r in range(W):
        for t in range(T):
            for pe in range(W):
                s = slot.get((pe, r, t), -1)
                assert res["slotmap"][r, t, pe] == s
                if s < 0:
                    continue
                assert res["recv_x"][pe, s].tobytes() == xb[r, t].tobytes()
                meta = res["recv_meta"][pe, s]
                assert (meta[0], meta[1]) == (r, t)
                for j in range(k):
                    e = int(idx[r, t, j])
                    assert meta[3 + j] == ((e % nEpr) if (e >= 0 and e // nEpr == pe) else -1)
                if w is None:
                    assert float(res["wsum"][r, t, pe]) == 1.0
                else:  # float32 fold in topk order, exactly
                    s32 = Fraction(0)
                    for j in range(k):
                        e = int(idx[r, t, j])
                        if e >= 0 and e // nEpr == pe:
                            s32 = P.round_fraction_to_f32(s32 + Fraction(float(w[r, t, j])))
                    assert Fraction(float(res["wsum"][r, t, pe])) == s32


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(problems())
def test_combine_matches_the_exact_fold(prob):
    cfg, xb, idx, w = prob
    if cfg["dtype"] != 0:  # the bf16 leg on bf16 payloads: y = the dispatched rows
        cfg = dict(cfg, dtype=0, hiddenDim=8)
        xb = P.random_payload(np.random.default_rng(int(idx.sum()) & 0xFFFF), xb.shape[:2] + (8,), 0)
    W, T, h = cfg["worldSize"], cfg["maxTokPerRank"], cfg["hiddenDim"]
    res = oracle.dispatch(cfg, xb, idx, w)
    out = oracle.combine(cfg, res["recv_x"], res["slotmap"], res["wsum"])
    yv = P.bf16_bits_to_f64(res["recv_x"])
    outv = P.bf16_bits_to_f64(out)
    for r in range(W):
        for t in range(T):
            for i in range(h):
                acc = Fraction(0)
                for pe in range(W):
                    s = int(res["slotmap"][r, t, pe])
                    if s >= 0:
                        prod = Fraction(float(res["wsum"][r, t, pe])) * Fraction(float(yv[pe, s, i]))
                        acc = P.round_fraction_to_f32(prod + acc)
                want = P.round_fraction_to_bf16(acc)
                assert Fraction(float(outv[r, t, i])) == want
