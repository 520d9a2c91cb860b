"""The README's usage example runs as written on the GPU (the full main
workload's buffers, about 5 GB), with a device error word of 0."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.gpu
def test_readme_example_runs():
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, flags=re.S)
    assert blocks, "README has no python example"
    exec(compile(blocks[0], "README.md example", "exec"), {})
