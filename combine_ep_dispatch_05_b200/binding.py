"""ctypes binding of libep_b200.so (include/ep.h): the same entry points, by
name, with argument marshalling only. Every step of dispatch and combine runs
in the library's CUDA kernels; if the library is missing, importing this module
fails instead of falling back to anything else.

Buffers may be passed as integers (device addresses) or as objects with a
``data_ptr()`` method (torch tensors); streams as integers, ``None`` (the legacy
default stream) or objects with a ``cuda_stream`` attribute.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# EP_B200_LIBRARY=debug loads the bounds-checking build (libep_b200_debug.so).
LIB_PATH = os.path.join(_PKG, "libep_b200_debug.so" if os.environ.get("EP_B200_LIBRARY") == "debug"
                        else "libep_b200.so")

EP_BF16, EP_FP32, EP_FP8, EP_FP4X2 = 0, 1, 2, 3
EP_OK = 0
EP_ERR_INVALID, EP_ERR_UNSUPPORTED, EP_ERR_NOMEM, EP_ERR_CUDA = -1, -2, -3, -4
EP_ERR_STATE, EP_ERR_ALIGN, EP_ERR_DEVICE = -5, -6, -7
EP_DEVERR_EXPERT_RANGE, EP_DEVERR_TIMEOUT, EP_DEVERR_CAPACITY, EP_DEVERR_BOUNDS = 1, 2, 4, 8

EXPORTED = ("ep_cfg_check", "ep_plan_query", "ep_plan_create", "ep_plan_destroy", "ep_plan_info",
            "ep_dispatch", "ep_combine", "ep_plan_check_error", "ep_last_error", "ep_dispatch_noalloc",
            "ep_dispatch_scaled", "ep_comm_create", "ep_comm_handle", "ep_comm_connect", "ep_comm_info",
            "ep_comm_dispatch", "ep_comm_combine", "ep_comm_check_error", "ep_comm_destroy",
            "ep_comm_barrier_selftest")
EP_SYNC_DEVICE, EP_SYNC_HOST = 0, 1
EP_ERR_PEER = -8
EP_COMM_HANDLE_BYTES = 256
EP_MAX_SCALE_WORDS = 4096
EP_NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024


class EpCfg(ctypes.Structure):
    _fields_ = [("worldSize", ctypes.c_int32), ("hiddenDim", ctypes.c_int32),
                ("maxTokPerRank", ctypes.c_int32), ("numExpertPerRank", ctypes.c_int32),
                ("numExpertPerToken", ctypes.c_int32), ("maxRecv", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("useWeights", ctypes.c_int32)]


class EpPlanInfo(ctypes.Structure):
    _fields_ = [("maxRecv", ctypes.c_int32), ("metaFields", ctypes.c_int32),
                ("rowBytes", ctypes.c_int64), ("tokenBytes", ctypes.c_int64),
                ("recvXBytes", ctypes.c_int64), ("recvMetaBytes", ctypes.c_int64),
                ("scratchBytes", ctypes.c_int64), ("countTile", ctypes.c_int32),
                ("numTiles", ctypes.c_int32), ("scatterBlocks", ctypes.c_int32),
                ("scatterWarps", ctypes.c_int32), ("scatterStages", ctypes.c_int32),
                ("scatterChunkBytes", ctypes.c_int32), ("combineBlocks", ctypes.c_int32),
                ("combineWarps", ctypes.c_int32), ("device", ctypes.c_int32),
                ("numSMs", ctypes.c_int32), ("scatterMode", ctypes.c_int32),
                ("scatterPend", ctypes.c_int32), ("combineDtype", ctypes.c_int32),
                ("combineHidden", ctypes.c_int32), ("combineRowBytes", ctypes.c_int64),
                ("yBytes", ctypes.c_int64), ("outBytes", ctypes.c_int64),
                ("dispatchFused", ctypes.c_int32), ("combineLoadBytes", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}


class EpCommInfo(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("worldSize", ctypes.c_int32), ("sync", ctypes.c_int32),
                ("maxRecv", ctypes.c_int32), ("metaFields", ctypes.c_int32), ("maxLanding", ctypes.c_int32),
                ("rowBytes", ctypes.c_int64), ("combineRowBytes", ctypes.c_int64),
                ("recvX", ctypes.c_void_p), ("recvMeta", ctypes.c_void_p), ("recvCount", ctypes.c_void_p),
                ("sharedBytes", ctypes.c_int64), ("localBytes", ctypes.c_int64),
                ("scatterBlocks", ctypes.c_int32), ("scatterWarps", ctypes.c_int32),
                ("scatterStages", ctypes.c_int32), ("combineBlocks", ctypes.c_int32),
                ("combineWarps", ctypes.c_int32), ("device", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}


HOST_BARRIER = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p)


class EpError(RuntimeError):
    def __init__(self, code: int, where: str, msg: str):
        super().__init__(f"{where} failed ({code}): {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m combine_ep_dispatch_05_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32 = ctypes.c_void_p, ctypes.c_int
    cfgp, infop = ctypes.POINTER(EpCfg), ctypes.POINTER(EpPlanInfo)
    sig = {
        "ep_cfg_check": ([cfgp], I32),
        "ep_plan_query": ([cfgp, infop], I32),
        "ep_plan_create": ([cfgp], P),
        "ep_plan_destroy": ([P], None),
        "ep_plan_info": ([P, infop], I32),
        "ep_dispatch": ([P, P, P, P, P, P, P, P], I32),
        "ep_combine": ([P, P, P, P], I32),
        "ep_plan_check_error": ([P], I32),
        "ep_last_error": ([], ctypes.c_char_p),
        "ep_dispatch_noalloc": ([cfgp, P, P, P, P, P, P, P], I32),
        "ep_dispatch_scaled": ([P, P, P, P, P, ctypes.c_int32, P, P, P, P, P], I32),
        "ep_comm_create": ([cfgp, ctypes.c_int32, ctypes.c_int32, HOST_BARRIER, P], P),
        "ep_comm_handle": ([P, P], I32),
        "ep_comm_connect": ([P, P], I32),
        "ep_comm_info": ([P, ctypes.POINTER(EpCommInfo)], I32),
        "ep_comm_dispatch": ([P, P, P, P, P], I32),
        "ep_comm_combine": ([P, P, P, P], I32),
        "ep_comm_check_error": ([P], I32),
        "ep_comm_destroy": ([P], None),
        "ep_comm_barrier_selftest": ([ctypes.c_int32] * 4 + [P, P, P], I32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    return lib


_lib = _load()


def _addr(buf):
    if buf is None:
        return None
    if isinstance(buf, int):
        return buf
    return buf.data_ptr()


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _cfg(cfg) -> EpCfg:
    if isinstance(cfg, EpCfg):
        return cfg
    return EpCfg(**{n: int(cfg[n]) for n, _ in EpCfg._fields_})


def _check(rc: int, where: str) -> int:
    if rc < 0:
        raise EpError(rc, where, ep_last_error())
    return rc


def ep_last_error() -> str:
    return (_lib.ep_last_error() or b"").decode()


def ep_cfg_check(cfg) -> int:
    """Return EP_OK or a negative code (no exception); reason in ep_last_error()."""
    return _lib.ep_cfg_check(ctypes.byref(_cfg(cfg)))


def ep_plan_query(cfg) -> EpPlanInfo:
    info = EpPlanInfo()
    _check(_lib.ep_plan_query(ctypes.byref(_cfg(cfg)), ctypes.byref(info)), "ep_plan_query")
    return info


def ep_plan_create(cfg) -> int:
    h = _lib.ep_plan_create(ctypes.byref(_cfg(cfg)))
    if not h:
        raise EpError(EP_ERR_INVALID, "ep_plan_create", ep_last_error())
    return h


def ep_plan_destroy(plan: int) -> None:
    _lib.ep_plan_destroy(plan)


def ep_plan_info(plan: int) -> EpPlanInfo:
    info = EpPlanInfo()
    _check(_lib.ep_plan_info(plan, ctypes.byref(info)), "ep_plan_info")
    return info


def ep_dispatch(plan: int, x, topk_idx, topk_w, recv_x, recv_meta, recv_count, stream=None) -> int:
    return _check(_lib.ep_dispatch(plan, _addr(x), _addr(topk_idx), _addr(topk_w), _addr(recv_x),
                                   _addr(recv_meta), _addr(recv_count), _stream(stream)),
                  "ep_dispatch")


def ep_dispatch_scaled(plan: int, x, topk_idx, topk_w, scales, scale_words: int, recv_x, recv_meta,
                       recv_scales, recv_count, stream=None) -> int:
    return _check(_lib.ep_dispatch_scaled(plan, _addr(x), _addr(topk_idx), _addr(topk_w), _addr(scales),
                                          int(scale_words), _addr(recv_x), _addr(recv_meta),
                                          _addr(recv_scales), _addr(recv_count), _stream(stream)),
                  "ep_dispatch_scaled")


def ep_combine(plan: int, y, out, stream=None) -> int:
    return _check(_lib.ep_combine(plan, _addr(y), _addr(out), _stream(stream)), "ep_combine")


def ep_dispatch_noalloc(cfg, x, topk_idx, topk_w, recv_x, recv_meta, recv_count, stream=None) -> int:
    """Plan-free dispatch whose scratch is a fixed device array (no allocation);
    see include/ep.h for its limit and its sharing rules."""
    return _check(_lib.ep_dispatch_noalloc(ctypes.byref(_cfg(cfg)), _addr(x), _addr(topk_idx),
                                           _addr(topk_w), _addr(recv_x), _addr(recv_meta),
                                           _addr(recv_count), _stream(stream)),
                  "ep_dispatch_noalloc")


def ep_plan_check_error(plan: int) -> int:
    return _check(_lib.ep_plan_check_error(plan), "ep_plan_check_error")


def library_path() -> str:
    return LIB_PATH


# ------------------------------------------------------------ ranks in processes
# The host barrier functions handed to the library must outlive the
# communicator: they are kept here by communicator handle.
_barriers: dict = {}


def ep_comm_create(cfg, rank: int, sync: int = EP_SYNC_DEVICE, barrier=None) -> int:
    """Rank `rank` of a communicator (include/ep_comm.h). barrier: for
    EP_SYNC_HOST, a function of no arguments that returns once every rank has
    called it and raises when that cannot happen (e.g. a torch.distributed
    barrier with a timeout)."""
    cb = None
    if barrier is not None:
        def _call(_ctx):
            try:
                barrier()
                return 0
            except Exception:  # a rank did not arrive: the library abandons the call
                return 1
        cb = HOST_BARRIER(_call)
    h = _lib.ep_comm_create(ctypes.byref(_cfg(cfg)), int(rank), int(sync),
                            cb if cb is not None else HOST_BARRIER(), None)
    if not h:
        raise EpError(EP_ERR_INVALID, "ep_comm_create", ep_last_error())
    _barriers[h] = cb
    return h


def ep_comm_handle(comm: int) -> bytes:
    buf = ctypes.create_string_buffer(EP_COMM_HANDLE_BYTES)
    _check(_lib.ep_comm_handle(comm, buf), "ep_comm_handle")
    return buf.raw


def ep_comm_connect(comm: int, records) -> int:
    """records: every rank's ep_comm_handle bytes, in rank order."""
    blob = b"".join(bytes(r) for r in records)
    buf = ctypes.create_string_buffer(blob, len(blob))
    return _check(_lib.ep_comm_connect(comm, buf), "ep_comm_connect")


def ep_comm_info(comm: int) -> EpCommInfo:
    info = EpCommInfo()
    _check(_lib.ep_comm_info(comm, ctypes.byref(info)), "ep_comm_info")
    return info


def ep_comm_dispatch(comm: int, x, topk_idx, topk_w, stream=None) -> int:
    return _check(_lib.ep_comm_dispatch(comm, _addr(x), _addr(topk_idx), _addr(topk_w), _stream(stream)),
                  "ep_comm_dispatch")


def ep_comm_combine(comm: int, y, out, stream=None) -> int:
    return _check(_lib.ep_comm_combine(comm, _addr(y), _addr(out), _stream(stream)), "ep_comm_combine")


def ep_comm_check_error(comm: int) -> int:
    return _check(_lib.ep_comm_check_error(comm), "ep_comm_check_error")


def ep_comm_barrier_selftest(W: int, rounds: int, absent_rank: int = -1, absent_from: int = 0):
    """Returns (barriers completed, error words, early reads), a list of W each."""
    arr = [(ctypes.c_int32 * W)() for _ in range(3)]
    _check(_lib.ep_comm_barrier_selftest(W, rounds, absent_rank, absent_from, *arr), "ep_comm_barrier_selftest")
    return tuple(list(a) for a in arr)


def ep_comm_destroy(comm: int) -> None:
    _lib.ep_comm_destroy(comm)
    _barriers.pop(comm, None)
