"""The usage example in README.md runs as written.

The first ```python block of the README is executed on cuda:0; its decode
output must be finite, of the query's shape, and the layer's device error word
must be clear (``layer.sync()`` inside the block raises otherwise).
"""
import math
import pathlib
import re

import pytest

pytestmark = pytest.mark.gpu

README = pathlib.Path(__file__).resolve().parent.parent / "README.md"


def _python_block() -> str:
    m = re.search(r"```python\n(.*?)```", README.read_text(), re.S)
    assert m, "README.md has no python block"
    return m.group(1)


def test_readme_example_runs(cuda_device):
    import torch

    ns: dict = {}
    exec(compile(_python_block(), str(README), "exec"), ns)
    o, dec = ns["o"], ns["dec"]
    assert o.is_cuda and tuple(o.shape) == tuple(dec["q"][0].shape)
    assert torch.isfinite(o.float()).all()
    assert math.isfinite(float(o.float().abs().max()))
