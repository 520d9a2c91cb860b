"""Host-side pieces of bench.py that need no GPU: the kernel-source hash that
keys the recorded ncu traffic, and the algorithmic byte counts."""
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


@pytest.fixture
def src_copy(tmp_path, monkeypatch):
    """A copy of the kernel sources, with bench reading from it."""
    for rel in bench.KERNEL_SOURCES + ["profiles/ncu_traffic.json"]:
        dst = tmp_path / rel
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    return tmp_path


def test_source_hash_ignores_comments_and_whitespace(src_copy):
    base = bench.source_hash()
    p = src_copy / bench.KERNEL_SOURCES[0]
    text = p.read_text()
    p.write_text("// a new comment line\n/* and a\n   block */\n" + text.replace(";\n", ";  \n", 3))
    assert bench.source_hash() == base


def test_source_hash_sees_code_changes(src_copy):
    base = bench.source_hash()
    p = src_copy / bench.KERNEL_SOURCES[1]
    p.write_text(p.read_text() + "\nconstexpr int kAnotherConstant = 1;\n")
    assert bench.source_hash() != base


def test_traffic_record_is_keyed_by_the_source_hash(src_copy):
    """The recorded traffic applies to the code and the launch geometry it was
    captured with and to nothing else: a code edit or another geometry makes
    bench report it as unknown."""
    import json
    geo = json.load(open(src_copy / "profiles" / "ncu_traffic.json"))["geometry"]["main"]
    rec = bench.ncu_traffic("ep_dispatch", "main", dict(geo))
    if rec is None:
        pytest.skip("the traffic record predates the current kernel code (profile again)")
    assert rec > 2.5e9
    assert bench.ncu_traffic("ep_dispatch", "main", dict(geo, scatterStages=geo["scatterStages"] + 1)) is None
    p = src_copy / bench.KERNEL_SOURCES[0]
    p.write_text(p.read_text() + "\nstatic int edited_code = 0;\n")
    assert bench.ncu_traffic("ep_dispatch", "main", dict(geo)) is None


def test_algorithmic_bytes_of_the_main_workload():
    """Dispatch and combine bytes from the formulas, at the seeded main
    routing's U = 173131 received rows."""
    wl = bench.get_workload("main")
    U, G, row, k = 173131, 8 * 4096, 14336, 8
    assert bench.dispatch_bytes(wl, U, G) == G * row + U * row + G * k * 4 * 2 + U * (3 + k) * 4 + 4 * 8
    assert bench.combine_bytes(wl, U) == U * row + G * row + U * 8
