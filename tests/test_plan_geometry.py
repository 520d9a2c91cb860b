"""Host-only plan sizing (ep_plan_query) over many random configurations:
the geometry the kernels are launched with keeps the invariants their index
arithmetic relies on. No GPU is needed; the query models a 148-SM B200."""
import numpy as np
import pytest

SMEM_OPTIN = 227 * 1024


@pytest.fixture(scope="module")
def ep():
    from combine_ep_dispatch_05_b200 import build
    build.build()
    import combine_ep_dispatch_05_b200 as m
    return m


def random_cfgs(n, seed):
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        dtype = int(rng.integers(0, 4))
        es = {0: 2, 1: 4, 2: 1, 3: 1}[dtype]
        W = int(rng.integers(1, 33))
        T = int(rng.choice([1, 2, 7, 64, 300, 512, 513, 1024, 4096]))
        k = int(rng.integers(1, 33))
        # hidden sizes whose rows are whole 16-byte vectors, from 16 bytes to 128 KB
        row = 16 * int(rng.integers(1, 8193))
        h = row // es
        nEpr = int(rng.integers(1, 65))
        maxRecv = W * T * int(rng.choice([1, 1, 2]))
        if W * maxRecv > (1 << 31) - 1:
            continue
        out.append(dict(worldSize=W, hiddenDim=h, maxTokPerRank=T, numExpertPerRank=nEpr,
                        numExpertPerToken=k, maxRecv=maxRecv, dtype=dtype, useWeights=int(rng.integers(0, 2))))
    return out


def scatter_smem(warps, stages, chunk_stride):
    head = (warps * stages * (8 + 8) + 127) & ~127
    return head + warps * stages * chunk_stride


@pytest.mark.parametrize("fused", ["0", "1"], ids=["default", "fused-enabled"])
def test_random_plan_geometry(ep, fused, monkeypatch):
    monkeypatch.setenv("EP_DISPATCH_FUSED", fused)
    for cfg in random_cfgs(400, 7 + 505 * int(fused)):
        assert ep.ep_cfg_check(cfg) == 0, (cfg, ep.ep_last_error())
        info = ep.ep_plan_query(cfg)
        W, T, k = cfg["worldSize"], cfg["maxTokPerRank"], cfg["numExpertPerToken"]
        G = W * T
        es = {0: 2, 1: 4, 2: 1, 3: 1}[cfg["dtype"]]
        row = cfg["hiddenDim"] * es
        assert info.rowBytes == row and info.maxRecv == cfg["maxRecv"]
        assert info.metaFields == 3 + k
        assert info.numTiles == -(-G // info.countTile)
        # row pieces: 16-byte multiples that cover the row
        chunk = info.scatterChunkBytes
        assert chunk % 16 == 0 and 16 <= chunk <= max(row, 16)
        assert -(-row // chunk) * chunk >= row
        stride = (chunk + 127) & ~127
        assert info.scatterStages >= 2 and info.scatterWarps >= 1
        assert scatter_smem(info.scatterWarps, info.scatterStages, stride) <= SMEM_OPTIN
        if info.dispatchFused:  # one launch: at most 64 tokens a block, at most one block a token
            assert fused == "1"
            assert info.scatterBlocks <= G and -(-G // info.scatterBlocks) <= 64
        # scratch holds at least the routing table and the token masks
        assert info.scratchBytes >= G * W * 8 + G * 4
        # the combine leg
        chid = 2 * cfg["hiddenDim"] if cfg["dtype"] == 3 else cfg["hiddenDim"]
        assert info.combineHidden == chid
        assert info.combineRowBytes == chid * (4 if cfg["dtype"] == 1 else 2)
        assert info.yBytes == W * cfg["maxRecv"] * info.combineRowBytes
        assert info.outBytes == G * info.combineRowBytes
