"""The bounds-checking build (libep_b200_debug.so), which stands in for a
memory checker: every copy's addresses are checked against their buffers, and
an access outside one is skipped and reported as EP_DEVERR_BOUNDS. Each case
runs in a fresh process, since the binding picks its library at import."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["clean", "shrunk"])
def test_bounds_checking_build(mode):
    from combine_ep_dispatch_05_b200 import build
    build.build()
    env = dict(os.environ, EP_B200_LIBRARY="debug")
    env.pop("EP_TEST_BOUNDS_ROWS", None)
    out = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_bounds_run.py"), mode],
                         env=env, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0 and out.stdout.strip().endswith("ok"), out.stdout[-3000:] + out.stderr[-3000:]


def test_binding_loads_the_debug_build_on_request():
    """Without a GPU too: the environment switch picks the other library, and
    a missing one is an import error, not a fallback."""
    code = ("import combine_ep_dispatch_05_b200.binding as b; print(b.LIB_PATH)")
    env = dict(os.environ, EP_B200_LIBRARY="debug")
    out = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, cwd=ROOT)
    assert out.stdout.strip().endswith("libep_b200_debug.so"), out.stderr
