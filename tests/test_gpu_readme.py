"""The README's usage example runs as written on the GPU and gives sane
results (shapes, dtypes, a round-trip error of the codec's size)."""

import os
import re

import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_runs():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, re.S)
    assert len(blocks) == 1
    env = {}
    exec(compile(blocks[0], "README.md", "exec"), env)
    x = env["x"]
    for name in ("xhat", "xhat_d"):
        xh = env[name]
        assert xh.shape == x.shape and xh.dtype == torch.float16
        err = ((xh.float() - x.float()).norm(dim=-1) / x.float().norm(dim=-1)).mean().item()
        assert err < 0.15, (name, err)   # int4 G16 on N(0, 1) data: about 0.07
    assert env["codes_d"].dtype == torch.uint8 and env["scales_d"].dtype == torch.float16
