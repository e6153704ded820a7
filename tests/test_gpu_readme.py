"""The usage example in README.md runs as written (on the GPU) and its results are sane."""
import os
import re

import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_runs(cuda_lib):
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, flags=re.S)
    assert len(blocks) == 1
    env = {}
    exec(compile(blocks[0], "README.md", "exec"), env)   # noqa: S102 - the repository's own documentation
    torch.cuda.synchronize()
    out, state, grads, leaves = env["out"], env["state"], env["grads"], env["leaves"]
    assert out.shape == (1, 4096, 16, 128) and state.shape == (1, 16, 128, 128)
    assert torch.isfinite(out).all() and torch.isfinite(state).all()
    assert len(grads) == 6 and all(torch.isfinite(g).all() for g in grads[:5])
    assert all(t.grad is not None and t.grad.dtype == t.dtype for t in leaves)
