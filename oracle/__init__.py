"""CPU oracle for MoE expert-parallel dispatch / combine -- test infrastructure.

Only the tests, the smoke check and the CPU-baseline leg of the bench may
import this package. The product path (the CUDA library and its binding) never
imports, links or calls it.

The arithmetic lives in ``ep_oracle.c`` (plain C, compiled here with ``gcc -O2
-ffp-contract=off``); this module only builds it and marshals numpy arrays
through ctypes. ``load_omp()`` gives the same source built with OpenMP, whose
results are identical, for timing the oracle on all host cores.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ep_oracle.c")
_LIB = os.path.join(_HERE, "libep_oracle.so")
_lock = threading.Lock()
_lib = None

STATUS_EXPERT_RANGE = 1


class OracleCfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "worldSize", "hiddenDim", "maxTokPerRank", "numExpertPerRank",
        "numExpertPerToken", "maxRecv", "dtype", "useWeights")]


_LIB_OMP = os.path.join(_HERE, "libep_oracle_omp.so")
_lib_omp = None
_FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def _compile(out: str, extra: list, force: bool) -> str:
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(_SRC):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_FLAGS, *extra, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile ep_oracle.c into shared libraries next to it: the
    single-threaded build (returned) and the OpenMP build."""
    _compile(_LIB_OMP, ["-fopenmp"], force)
    return _compile(_LIB, [], force)


def _bind(lib):
    P = ctypes.c_void_p
    cfgp = ctypes.POINTER(OracleCfg)
    lib.oracle_dispatch.argtypes = [cfgp, P, P, P, P, P, P, P, P]
    lib.oracle_dispatch.restype = ctypes.c_int
    lib.oracle_dispatch_scaled.argtypes = [cfgp, P, P, P, P, ctypes.c_int64, P, P, P, P, P, P]
    lib.oracle_dispatch_scaled.restype = ctypes.c_int
    lib.oracle_combine.argtypes = [cfgp, P, P, P, P]
    lib.oracle_combine.restype = ctypes.c_int
    lib.oracle_recv_capacity.argtypes = [cfgp]
    lib.oracle_recv_capacity.restype = ctypes.c_int
    lib.oracle_f32_to_bf16.argtypes = [P, P, ctypes.c_int64]
    lib.oracle_f32_to_bf16.restype = None
    lib.oracle_bf16_to_f32.argtypes = [P, P, ctypes.c_int64]
    lib.oracle_bf16_to_f32.restype = None
    lib.oracle_threads.argtypes = []
    lib.oracle_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
    return _lib


def load_omp():
    """The OpenMP build of the same source: same results, all host cores
    (OMP_NUM_THREADS caps them). Pass it as ``lib=``."""
    global _lib_omp
    with _lock:
        if _lib_omp is None:
            build()
            _lib_omp = _bind(ctypes.CDLL(_LIB_OMP))
    return _lib_omp


def threads(lib=None) -> int:
    """Threads a call of this build may use (1 for the single-threaded one)."""
    return int((lib or _load()).oracle_threads())


def load_library(path: str):
    """Bind another build of ep_oracle.c (tests plant mistakes in a copy of the
    source to check that the pins catch them); pass the result as ``lib=``."""
    return _bind(ctypes.CDLL(path))


def _cfg(cfg: dict) -> OracleCfg:
    return OracleCfg(**{k: int(cfg[k]) for k in (
        "worldSize", "hiddenDim", "maxTokPerRank", "numExpertPerRank",
        "numExpertPerToken", "maxRecv", "dtype", "useWeights")})


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def recv_capacity(cfg: dict) -> int:
    return int(cfg["maxRecv"]) or int(cfg["worldSize"]) * int(cfg["maxTokPerRank"])


# Payload dtypes (numbering of the design page's EpDType): the numpy type in
# which tests hold one dispatched element, and its size in bytes.
PAYLOAD_NP = {0: np.uint16, 1: np.float32, 2: np.uint8, 3: np.uint8}


def payload_np(cfg: dict):
    return PAYLOAD_NP[int(cfg["dtype"])]


def combine_hidden(cfg: dict) -> int:
    """Elements of a combine row: 2 * hiddenDim for fp4x2 (packed pairs)."""
    h = int(cfg["hiddenDim"])
    return 2 * h if int(cfg["dtype"]) == 3 else h


def combine_np(cfg: dict):
    """float32 for an fp32 plan; bf16 bits (uint16) otherwise."""
    return np.float32 if int(cfg["dtype"]) == 1 else np.uint16


def dispatch(cfg: dict, x: np.ndarray, topk_idx: np.ndarray, topk_w, recv_x=None, recv_meta=None,
             lib=None, scales=None, recv_scales=None):
    """Run the oracle dispatch. Returns a dict with recv_x, recv_meta,
    recv_count, slotmap, wsum and status (0, or STATUS_EXPERT_RANGE).

    ``recv_x`` / ``recv_meta`` may be passed pre-filled (e.g. with a canary) to
    observe which entries the oracle leaves untouched.
    """
    lib = lib or _load()
    c = _cfg(cfg)
    W, T, h, k = c.worldSize, c.maxTokPerRank, c.hiddenDim, c.numExpertPerToken
    R = recv_capacity(cfg)
    pt = payload_np(cfg)
    x = np.ascontiguousarray(x).view(pt).reshape(W, T, h)
    idx = np.ascontiguousarray(topk_idx, dtype=np.int32).reshape(W, T, k)
    w = None if topk_w is None else np.ascontiguousarray(topk_w, dtype=np.float32).reshape(W, T, k)
    if recv_x is None:
        recv_x = np.zeros((W, R, h), dtype=pt)
    if recv_meta is None:
        recv_meta = np.zeros((W, R, 3 + k), dtype=np.int32)
    recv_x = recv_x.view(pt)
    assert recv_x.shape == (W, R, h) and recv_x.flags.c_contiguous
    assert recv_meta.shape == (W, R, 3 + k) and recv_meta.dtype == np.int32
    recv_count = np.zeros(W, dtype=np.int32)
    slotmap = np.empty((W, T, W), dtype=np.int32)
    wsum = np.empty((W, T, W), dtype=np.float32)
    if scales is None:
        rc = lib.oracle_dispatch(ctypes.byref(c), _ptr(x), _ptr(idx), _ptr(w), _ptr(recv_x),
                                 _ptr(recv_meta), _ptr(recv_count), _ptr(slotmap), _ptr(wsum))
    else:
        sw = np.ascontiguousarray(scales).view(np.uint32).reshape(W, T, -1)
        if recv_scales is None:
            recv_scales = np.zeros((W, R, sw.shape[-1]), dtype=np.uint32)
        recv_scales = recv_scales.view(np.uint32)
        assert recv_scales.shape == (W, R, sw.shape[-1]) and recv_scales.flags.c_contiguous
        rc = lib.oracle_dispatch_scaled(ctypes.byref(c), _ptr(x), _ptr(idx), _ptr(w), _ptr(sw),
                                        sw.shape[-1], _ptr(recv_x), _ptr(recv_meta), _ptr(recv_scales),
                                        _ptr(recv_count), _ptr(slotmap), _ptr(wsum))
    if rc < 0:
        raise ValueError(f"oracle_dispatch rejected its arguments (rc={rc})")
    return dict(recv_x=recv_x, recv_meta=recv_meta, recv_count=recv_count,
                slotmap=slotmap, wsum=wsum, status=rc, recv_scales=recv_scales)


def combine(cfg: dict, y: np.ndarray, slotmap: np.ndarray, wsum: np.ndarray, lib=None,
            out: np.ndarray = None) -> np.ndarray:
    """Run the oracle combine; returns out, shape (W, T, combine_hidden): bf16
    bits (uint16), or float32 for an fp32 plan. ``out`` may be passed
    pre-allocated (every row is written)."""
    lib = lib or _load()
    c = _cfg(cfg)
    W, T = c.worldSize, c.maxTokPerRank
    h = combine_hidden(cfg)
    R = recv_capacity(cfg)
    ct = combine_np(cfg)
    y = np.ascontiguousarray(y).view(ct).reshape(W, R, h)
    slotmap = np.ascontiguousarray(slotmap, dtype=np.int32).reshape(W, T, W)
    wsum = np.ascontiguousarray(wsum, dtype=np.float32).reshape(W, T, W)
    if out is None:
        out = np.empty((W, T, h), dtype=ct)
    assert out.shape == (W, T, h) and out.dtype == ct and out.flags.c_contiguous
    rc = lib.oracle_combine(ctypes.byref(c), _ptr(y), _ptr(slotmap), _ptr(wsum), _ptr(out))
    if rc < 0:
        raise ValueError(f"oracle_combine rejected its arguments (rc={rc})")
    return out


def f32_to_bf16(a: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or _load()
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    lib.oracle_f32_to_bf16(_ptr(a), _ptr(out), a.size)
    return out


def bf16_to_f32(a: np.ndarray, lib=None) -> np.ndarray:
    lib = lib or _load()
    a = np.ascontiguousarray(a, dtype=np.uint16)
    out = np.empty(a.shape, dtype=np.float32)
    lib.oracle_bf16_to_f32(_ptr(a), _ptr(out), a.size)
    return out
