"""Seeded synthetic workloads for MoE expert-parallel dispatch / combine.

This module only draws random inputs. It holds none of the dispatch or combine
arithmetic (no destination mapping, no dedup, no slot order, no reduction), so
that both the CPU oracle and the CUDA path can consume the same inputs without
sharing any of the method's code.

Workloads follow the shapes the pages measure:

* ``tiny``     -- W=2, 8 tokens/rank, hidden 256, 4 experts/rank, topk 2.
* ``pr599``    -- W=4, ct=512, hidden 7168, 8 experts/rank, topk 6: the shape of
                  the dispatch measurement in mori PR #599 ("Perf/ep disp 1250
                  ship", Results section).
* ``main``     -- W=8, ct=4096, hidden 7168, 32 experts/rank (256), topk 8: the
                  EP8 hidden-7168 topk-8 shape of the MORI JIT v2 design page, §8.
* ``latency1`` / ``latency8`` -- W=8, hidden 2048, 8 experts/rank, topk 6,
                  maxTokPerRank 512, maxRecv 4096, only 1 / 8 live tokens per rank,
                  no weights: the generated-source example of the design page §3.3
                  and the ct=1/ct=8 correctness shapes of PR #599.
* ``skewed``   -- the ``main`` shape with expert popularity p_e ~ (e+1)^-1.2 (Zipf
                  s=1.2), so destination rank 0 is hot.

Draw order per workload, from ``numpy.random.Generator(PCG64(seed))``:
topk expert ids, then gating logits, then the hidden rows ``x``.

* Uniform routing: per live token, an argsort of E uniforms gives a random
  permutation of the experts; its first ``k`` entries are the token's ids, in
  that order (k distinct experts).
* Zipf routing: Gumbel-top-k without replacement on log p_e; ids in descending
  key order.
* Weights: softmax over the token's ``k`` N(0,1) logits, computed in float32.
* ``x`` ~ N(0,1) in float32, rounded to bfloat16 (round-to-nearest-even, done by
  torch's dtype conversion); returned as the raw uint16 bit patterns.
* Rows ``t >= ct`` carry expert id -1 in every topk position (absent tokens) and
  weight 0.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "make_inputs", "workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    W: int            # worldSize: virtual expert-parallel ranks
    max_tok: int      # maxTokPerRank
    ct: int           # live tokens per rank in this call (rows >= ct are absent)
    h: int            # hiddenDim (bf16 elements per row)
    n_epr: int        # numExpertPerRank
    k: int            # numExpertPerToken (topk)
    routing: str      # "uniform" or "zipf1.2"
    use_weights: bool
    max_recv: int     # per-destination receive capacity (0 means W*max_tok)
    seed: int

    @property
    def E(self) -> int:
        return self.W * self.n_epr

    def cfg(self) -> dict:
        """EpCfg field values (dtype 0 = bf16)."""
        return dict(worldSize=self.W, hiddenDim=self.h, maxTokPerRank=self.max_tok,
                    numExpertPerRank=self.n_epr, numExpertPerToken=self.k,
                    maxRecv=self.max_recv, dtype=0, useWeights=int(self.use_weights))

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny", W=2, max_tok=8, ct=8, h=256, n_epr=4, k=2, routing="uniform",
                 use_weights=True, max_recv=16, seed=0),
        Workload("pr599", W=4, max_tok=512, ct=512, h=7168, n_epr=8, k=6, routing="uniform",
                 use_weights=True, max_recv=2048, seed=1),
        Workload("main", W=8, max_tok=4096, ct=4096, h=7168, n_epr=32, k=8, routing="uniform",
                 use_weights=True, max_recv=32768, seed=2),
        Workload("latency1", W=8, max_tok=512, ct=1, h=2048, n_epr=8, k=6, routing="uniform",
                 use_weights=False, max_recv=4096, seed=3),
        Workload("latency8", W=8, max_tok=512, ct=8, h=2048, n_epr=8, k=6, routing="uniform",
                 use_weights=False, max_recv=4096, seed=3),
        Workload("skewed", W=8, max_tok=4096, ct=4096, h=7168, n_epr=32, k=8, routing="zipf1.2",
                 use_weights=True, max_recv=32768, seed=4),
    ]
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def _draw_ids(rng: np.random.Generator, wl: Workload) -> np.ndarray:
    """Expert ids of the live tokens, shape (W, ct, k), int32."""
    E, k = wl.E, wl.k
    shape = (wl.W, wl.ct, E)
    if wl.routing == "uniform":
        u = rng.random(shape)
        ids = np.argsort(u, axis=-1, kind="stable")[..., :k]
    elif wl.routing.startswith("zipf"):
        s = float(wl.routing[4:])
        logp = -s * np.log(np.arange(1, E + 1, dtype=np.float64))
        logp -= np.log(np.exp(logp).sum())
        g = -np.log(-np.log(rng.random(shape)))
        key = logp[None, None, :] + g
        ids = np.argsort(-key, axis=-1, kind="stable")[..., :k]
    else:
        raise ValueError(f"unknown routing {wl.routing!r}")
    return ids.astype(np.int32)


def _softmax_f32(logits: np.ndarray) -> np.ndarray:
    z = logits.astype(np.float32)
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z, dtype=np.float32)
    return (e / e.sum(axis=-1, keepdims=True, dtype=np.float32)).astype(np.float32)


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (RNE, via torch's conversion); return uint16 bits."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def make_inputs(wl: Workload, with_x: bool = True, x_rows: Optional[int] = None) -> dict:
    """Return the seeded inputs of one call.

    Keys: ``x`` (uint16 bf16 bits, (W, max_tok, h)) unless ``with_x`` is False,
    ``topk_idx`` (int32, (W, max_tok, k)), ``topk_w`` (float32, same shape, or
    None when the workload runs without weights).
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    W, T, k = wl.W, wl.max_tok, wl.k
    idx = np.full((W, T, k), -1, dtype=np.int32)
    idx[:, :wl.ct, :] = _draw_ids(rng, wl)
    logits = rng.standard_normal((W, wl.ct, k), dtype=np.float32)
    w = np.zeros((W, T, k), dtype=np.float32)
    w[:, :wl.ct, :] = _softmax_f32(logits)
    out = {"topk_idx": idx, "topk_w": w if wl.use_weights else None}
    if with_x:
        rows = T if x_rows is None else x_rows
        xf = rng.standard_normal((W, rows, wl.h), dtype=np.float32)
        x = np.zeros((W, T, wl.h), dtype=np.uint16)
        x[:, :rows, :] = bf16_bits_from_f32(xf)
        out["x"] = x
    return out
