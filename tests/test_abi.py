"""The C ABI on a machine without a GPU: the library loads, exports every
entry point include/ep.h declares, its structs have the layout the header
gives, configuration checks follow the validity rules, and calls that need a
device fail with an error instead of crashing."""
import ctypes
import os
import re
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", "ep.h"), os.path.join(ROOT, "include", "ep_comm.h")]


@pytest.fixture(scope="module")
def ep():
    from combine_ep_dispatch_05_b200 import build
    build.build()
    import combine_ep_dispatch_05_b200 as mod
    return mod


def declared_functions():
    src = "".join(open(h).read() for h in HEADERS)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z_]+)\s*\(", src)))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ("ep_plan_create", "ep_dispatch", "ep_combine", "ep_plan_destroy", "ep_last_error",
              "ep_plan_info", "ep_plan_check_error", "ep_cfg_check", "ep_plan_query", "ep_comm_create",
              "ep_comm_handle", "ep_comm_connect", "ep_comm_dispatch", "ep_comm_combine", "ep_comm_destroy"):
        assert n in names


def test_library_exports_every_declared_symbol(ep):
    lib = ctypes.CDLL(ep.library_path())
    for n in declared_functions():
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", ep.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (ep_[a-z_]+)\b", out))
    assert set(declared_functions()) <= exported
    assert set(ep.binding.EXPORTED) == set(declared_functions())


def test_struct_layout_matches_header(ep, tmp_path):
    """sizeof/offsetof from a C compile of include/ep.h against the ctypes mirror."""
    fields = {"EpCfg": [n for n, _ in ep.EpCfg._fields_],
              "EpPlanInfo": [n for n, _ in ep.EpPlanInfo._fields_],
              "EpCommInfo": [n for n, _ in ep.EpCommInfo._fields_]}
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "ep_comm.h"', 'int main(void) {']
    for st, names in fields.items():
        lines.append(f'  printf("{st} size %zu\\n", sizeof({st}));')
        for n in names:
            lines.append(f'  printf("{st} {n} %zu\\n", offsetof({st}, {n}));')
    lines += ['  return 0;', '}']
    c = tmp_path / "layout.c"
    c.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)])
    rows = [l.split() for l in subprocess.check_output([str(exe)], text=True).splitlines()]
    for st, key, val in rows:
        cls = getattr(ep, st)
        if key == "size":
            assert ctypes.sizeof(cls) == int(val), st
        else:
            assert getattr(cls, key).offset == int(val), (st, key)


def test_header_compiles_as_plain_c_and_cpp(tmp_path):
    """The ABI header needs no CUDA header and compiles as C and C++."""
    for lang, comp in (("c", "gcc"), ("cpp", "g++")):
        f = tmp_path / f"inc.{lang}"
        f.write_text('#include "ep_comm.h"\nint main(void){ EpCfg c = {0}; return (int)sizeof(c) - 32; }\n')
        subprocess.check_call([comp, "-I", os.path.join(ROOT, "include"), str(f), "-o", str(tmp_path / lang)])
        assert subprocess.run([str(tmp_path / lang)]).returncode == 0


def _cfg(**kw):
    c = dict(worldSize=8, hiddenDim=7168, maxTokPerRank=4096, numExpertPerRank=32,
             numExpertPerToken=8, maxRecv=32768, dtype=0, useWeights=1)
    c.update(kw)
    return c


@pytest.mark.parametrize("kw,code", [
    (dict(), 0),
    (dict(maxRecv=0), 0),
    (dict(hiddenDim=7), -1),              # 14 bytes: not a multiple of 16
    (dict(hiddenDim=12), -1),             # 24 bytes
    (dict(hiddenDim=8), 0),               # 16 bytes
    (dict(numExpertPerToken=33), -1),     # topk must fit one warp
    (dict(numExpertPerToken=0), -1),
    (dict(worldSize=33), -1),             # worldSize must fit one warp
    (dict(worldSize=0), -1),
    (dict(maxRecv=32767), -1),            # capacity below the worst case
    (dict(maxTokPerRank=0), -1),
    (dict(numExpertPerRank=0), -1),
    (dict(dtype=2), 0),                   # fp8 transport: 7168-byte rows
    (dict(dtype=1), 0),                   # fp32 transport
    (dict(dtype=3, hiddenDim=3584), 0),   # fp4x2: hiddenDim counts bytes
    (dict(dtype=2, hiddenDim=8), -1),     # 8-byte fp8 rows: not a multiple of 16
    (dict(dtype=3, hiddenDim=24), -1),
    (dict(dtype=1, hiddenDim=4), 0),      # 16-byte fp32 rows
    (dict(dtype=9), -1),
    (dict(dtype=-1), -1),
    (dict(useWeights=2), -1),
    (dict(worldSize=32, maxTokPerRank=1 << 22, maxRecv=0), -1),  # flat index beyond int32
])
def test_cfg_check(ep, kw, code):
    assert ep.ep_cfg_check(_cfg(**kw)) == code
    if code:
        assert ep.ep_last_error()


def test_plan_query_sizes(ep):
    info = ep.ep_plan_query(_cfg(maxRecv=0))
    assert info.maxRecv == 8 * 4096
    assert info.metaFields == 11
    assert info.rowBytes == 14336
    assert info.tokenBytes == 8 * 4096 * 14336
    assert info.recvXBytes == 8 * 32768 * 14336
    assert info.recvMetaBytes == 8 * 32768 * 11 * 4
    assert info.numTiles == (8 * 4096 + info.countTile - 1) // info.countTile
    assert info.scatterChunkBytes % 16 == 0 and info.scatterStages >= 2
    big = ep.ep_plan_query(_cfg(hiddenDim=40000))
    assert big.scatterChunkBytes < big.rowBytes and big.scatterChunkBytes % 16 == 0
    assert (info.combineDtype, info.combineHidden, info.combineRowBytes) == (0, 7168, 14336)
    assert info.yBytes == info.recvXBytes and info.outBytes == info.tokenBytes


@pytest.mark.parametrize("dtype,h,row,chid,crow,cdt", [
    (0, 7168, 14336, 7168, 14336, 0),   # bf16 in, bf16 out
    (1, 7168, 28672, 7168, 28672, 1),   # fp32 in, fp32 out
    (2, 7168, 7168, 7168, 14336, 0),    # fp8 in, bf16 out
    (3, 3584, 3584, 7168, 14336, 0),    # fp4x2 in (h counts bytes), bf16 out over 2h
])
def test_plan_query_dtype_legs(ep, dtype, h, row, chid, crow, cdt):
    info = ep.ep_plan_query(_cfg(dtype=dtype, hiddenDim=h))
    assert info.rowBytes == row and info.tokenBytes == 8 * 4096 * row
    assert info.recvXBytes == 8 * 32768 * row
    assert (info.combineHidden, info.combineRowBytes, info.combineDtype) == (chid, crow, cdt)
    assert info.yBytes == 8 * 32768 * crow and info.outBytes == 8 * 4096 * crow


@pytest.mark.parametrize("kw,fused", [
    (dict(), 0),                                                       # main shape: 222 tokens a block
    (dict(maxTokPerRank=512, maxRecv=0), 1),                           # 4096 tokens: 28 a block
    (dict(maxTokPerRank=513, maxRecv=0), 1),
    (dict(worldSize=4, maxTokPerRank=512, numExpertPerRank=8, numExpertPerToken=6, maxRecv=0), 1),
    (dict(maxTokPerRank=512, numExpertPerToken=32, maxRecv=0), 1),     # topk 32
    (dict(worldSize=32, maxTokPerRank=512, numExpertPerToken=8, maxRecv=0), 0),  # 16384 tokens: 111 a block
    (dict(maxTokPerRank=1, maxRecv=0), 1),                             # 8 tokens: 8 blocks of one
    (dict(maxTokPerRank=512, maxRecv=0, dtype=1), 1),                  # fp32 rows of 28672 bytes
    (dict(maxTokPerRank=512, maxRecv=0, hiddenDim=100000), 1),         # rows copied in pieces
])
def test_plan_query_dispatch_form(ep, kw, fused, monkeypatch):
    """With EP_DISPATCH_FUSED=1, plans where no block owns more than 64 tokens
    take the one-launch fused dispatch (a grid of at most one block a token);
    the rest take route_count + scatter_rows. Both give identical results. By
    default the fused dispatch is off."""
    assert ep.ep_plan_query(_cfg(**kw)).dispatchFused == 0
    plain = ep.ep_plan_query(_cfg(**kw))
    monkeypatch.setenv("EP_DISPATCH_FUSED", "1")
    cfg = _cfg(**kw)
    info = ep.ep_plan_query(cfg)
    assert info.dispatchFused == fused
    G = cfg["worldSize"] * cfg["maxTokPerRank"]
    if fused:
        assert info.scatterBlocks == min(plain.scatterBlocks, G)
        assert -(-G // info.scatterBlocks) <= 64
        assert info.scratchBytes > plain.scratchBytes  # the blocks' published totals
    else:
        assert info.scatterBlocks == plain.scatterBlocks and info.scratchBytes == plain.scratchBytes


@pytest.mark.parametrize("kw,load", [
    (dict(), 32),                                               # output 470 MB, 14336-byte rows
    (dict(dtype=1), 32),                                        # fp32 leg, 28672-byte rows
    (dict(dtype=3, hiddenDim=3584), 32),                        # fp4x2 in, bf16 leg of 14336 bytes
    (dict(maxTokPerRank=2048, maxRecv=16384), 32),              # 235 MB
    (dict(maxTokPerRank=1024, maxRecv=8192), 16),               # 117 MB
    (dict(hiddenDim=2048), 16),                                 # 134 MB
    (dict(hiddenDim=14336, maxTokPerRank=2048, maxRecv=16384), 32),  # 470 MB from 16384 tokens
    (dict(worldSize=4, maxTokPerRank=512, numExpertPerRank=8, numExpertPerToken=6, maxRecv=0), 16),
    (dict(hiddenDim=7176), 16),                                 # 14352-byte rows: not a multiple of 32
])
def test_plan_query_combine_load_width(ep, kw, load, monkeypatch):
    """The combine reads y in 32-byte loads when its output is at least 192 MiB
    and its rows are a multiple of 32 bytes; EP_COMBINE_WIDE overrides the size
    rule but never the row rule."""
    cfg = _cfg(**kw)
    assert ep.ep_plan_query(cfg).combineLoadBytes == load
    row_ok = ep.ep_plan_query(cfg).combineRowBytes % 32 == 0
    monkeypatch.setenv("EP_COMBINE_WIDE", "1")
    assert ep.ep_plan_query(cfg).combineLoadBytes == (32 if row_ok else 16)
    monkeypatch.setenv("EP_COMBINE_WIDE", "0")
    assert ep.ep_plan_query(cfg).combineLoadBytes == 16


def test_entry_points_reject_without_crashing(ep):
    b = ep.binding
    assert b._lib.ep_dispatch(None, None, None, None, None, None, None, None) == b.EP_ERR_INVALID
    assert b._lib.ep_combine(None, None, None, None) == b.EP_ERR_INVALID
    assert b._lib.ep_plan_info(None, None) == b.EP_ERR_INVALID
    assert b._lib.ep_plan_check_error(None) == b.EP_ERR_INVALID
    for words in (0, -1, b.EP_MAX_SCALE_WORDS + 1):
        assert b._lib.ep_dispatch_scaled(None, None, None, None, None, words, None, None, None, None,
                                         None) == b.EP_ERR_INVALID
    b._lib.ep_plan_destroy(None)
    with pytest.raises(ep.EpError):
        ep.ep_plan_create(_cfg(hiddenDim=7))


def test_plan_create_without_device_fails_cleanly(ep):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(ep.EpError) as e:
        ep.ep_plan_create(_cfg(maxTokPerRank=8, maxRecv=0))
    assert "cuda" in str(e.value).lower()


def test_binding_fails_loudly_without_library(tmp_path):
    """No fallback: importing the binding without the built library raises."""
    pkg = tmp_path / "combine_ep_dispatch_05_b200"
    pkg.mkdir()
    src = os.path.join(ROOT, "combine_ep_dispatch_05_b200")
    for f in ("__init__.py", "binding.py"):
        (pkg / f).write_text(open(os.path.join(src, f)).read())
    code = textwrap.dedent("""
        import combine_ep_dispatch_05_b200 as ep
        try:
            ep.ep_dispatch
        except ImportError as e:
            print("IMPORTERROR", e)
    """)
    out = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True)
    assert "IMPORTERROR" in out.stdout and "libep_b200.so" in out.stdout


def test_graft_entry_build():
    """The build entry point compiles both libraries and loads the binding."""
    sys.path.insert(0, ROOT)
    import __graft_entry__
    __graft_entry__.build()


@pytest.mark.parametrize("which", ["topk_idx", "topk_w", "recv_meta", "recv_count", "x", "recv_x"])
def test_noalloc_rejects_misaligned_buffers_before_any_launch(ep, which):
    """ep_dispatch_noalloc checks alignment as ep_dispatch does, on the host,
    before it touches the device: a misaligned int32 / float buffer (4 bytes)
    or payload buffer (16 bytes) gives EP_ERR_ALIGN. The addresses here are
    never dereferenced, and on a machine without a GPU the call would fail with
    a CUDA error instead if it had got as far as the device."""
    from combine_ep_dispatch_05_b200 import binding as b
    bufs = {n: 0x10000 * (i + 1) for i, n in enumerate(
        ["x", "topk_idx", "topk_w", "recv_x", "recv_meta", "recv_count"])}
    bufs[which] += 2 if which not in ("x", "recv_x") else 8
    cfg = b._cfg(_cfg(maxTokPerRank=8, maxRecv=0))
    rc = b._lib.ep_dispatch_noalloc(ctypes.byref(cfg), bufs["x"], bufs["topk_idx"], bufs["topk_w"],
                                    bufs["recv_x"], bufs["recv_meta"], bufs["recv_count"], None)
    assert rc == b.EP_ERR_ALIGN
    assert "aligned" in ep.ep_last_error()


@pytest.mark.parametrize("dtype,h,blocks_per_sm", [(0, 7168, 1), (2, 7168, 2), (3, 3584, 4), (1, 7168, 1)])
def test_plan_query_blocks_per_sm(ep, dtype, h, blocks_per_sm):
    """Rows between 4 and 8 KB take two engines per block and stages few
    enough that two blocks share an SM's 228 KB (with each block's static
    shared memory and the 1 KB the system keeps); rows of at most 4 KB, three
    engines of 5 stages, as many blocks as fit; rows of 8 KB and more, one
    block."""
    info = ep.ep_plan_query(_cfg(dtype=dtype, hiddenDim=h))
    assert info.scatterBlocks == 148 * blocks_per_sm
    per_block = info.scatterWarps * info.scatterStages * ((info.scatterChunkBytes + 127) // 128 * 128)
    assert blocks_per_sm * (per_block + 128 + 2048 + 1024) <= 228 * 1024
