"""The README's Python example runs as written (on the 1024^2 x 512 C-arm
workload) and gives an image in [0, 1) and a non-zero gradient."""
import os
import re

import numpy as np
import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example():
    torch = pytest.importorskip("torch")
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    with open(os.path.join(ROOT, "README.md")) as f:
        text = f.read()
    block = re.search(r"## Use from Python\n\n((?:    .*\n|\n)+)", text).group(1)
    code = "\n".join(line[4:] for line in block.splitlines())
    scope = {}
    exec(compile(code, "README.md", "exec"), scope)
    torch.cuda.synchronize()
    img = scope["img"].cpu().numpy()
    grad = scope["grad"].cpu().numpy()
    assert np.all(img >= 0.0) and np.all(img < 1.0) and img.max() > 0.1
    assert np.all(np.isfinite(grad)) and np.abs(grad).max() > 0.0
