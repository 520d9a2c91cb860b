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
* Payload dtype (``dtype``, numbered as the design page's EpDType): 0 bf16 as
  above; 1 fp32 N(0,1); 2 fp8 e4m3 (N(0,1) converted by torch's float8_e4m3fn);
  3 fp4x2: N(0,1) rounded to the nearest e2m1 value (magnitudes 0, 0.5, 1, 1.5,
  2, 3, 4, 6 and a sign bit), two 4-bit codes per byte, the first element in
  the low nibble; ``h`` then counts bytes (2*h elements).
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
    dtype: int = 0    # payload: 0 bf16, 1 fp32, 2 fp8 (e4m3), 3 fp4x2 (h counts bytes)

    @property
    def E(self) -> int:
        return self.W * self.n_epr

    def cfg(self) -> dict:
        """EpCfg field values (dtype 0 = bf16)."""
        return dict(worldSize=self.W, hiddenDim=self.h, maxTokPerRank=self.max_tok,
                    numExpertPerRank=self.n_epr, numExpertPerToken=self.k,
                    maxRecv=self.max_recv, dtype=self.dtype, useWeights=int(self.use_weights))

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


_E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)


_E2M1_MID = (_E2M1[1:] + _E2M1[:-1]) / 2  # decision points between neighbours


def _e2m1_codes(v: np.ndarray) -> np.ndarray:
    """4-bit e2m1 codes (sign in bit 3) of the values nearest to v (a value
    exactly between two neighbours takes the smaller magnitude)."""
    code = np.searchsorted(_E2M1_MID, np.abs(v), side="left").astype(np.uint8)
    return code | (np.signbit(v).astype(np.uint8) << 3)


def payload_from_f32(xf: np.ndarray, dtype: int) -> np.ndarray:
    """The payload of float32 values in a dispatch dtype: uint16 bf16 bits,
    float32, uint8 e4m3 bytes, or uint8 bytes of packed e2m1 pairs (the last
    axis halves)."""
    if dtype == 0:
        return bf16_bits_from_f32(xf)
    if dtype == 1:
        return np.ascontiguousarray(xf, dtype=np.float32)
    if dtype == 2:
        import torch
        t = torch.from_numpy(np.ascontiguousarray(xf, dtype=np.float32)).to(torch.float8_e4m3fn)
        return t.view(torch.uint8).numpy()
    if dtype == 3:
        c = _e2m1_codes(xf)
        return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)
    raise ValueError(f"unknown dtype {dtype}")


def make_inputs(wl: Workload, with_x: bool = True, x_rows: Optional[int] = None) -> dict:
    """Return the seeded inputs of one call.

    Keys: ``x`` (the payload, (W, max_tok, h): uint16 bf16 bits, float32, or
    uint8 bytes for fp8 / fp4x2) unless ``with_x`` is False,
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
        n_el = 2 * wl.h if wl.dtype == 3 else wl.h  # fp4x2: h bytes hold 2*h elements
        xf = rng.standard_normal((W, rows, n_el), dtype=np.float32)
        pay = payload_from_f32(xf, wl.dtype)
        x = np.zeros((W, T, wl.h), dtype=pay.dtype)
        x[:, :rows, :] = pay
        out["x"] = x
    return out
