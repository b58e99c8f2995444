"""The README's Python example runs as written on the GPU, and its first
all-reduce equals the oracle's (needs a B200)."""
import os
import re

import numpy as np
import pytest
import torch

from oracle import oracle as O

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_python_example_runs():
    from quantized_precision_all_b200 import build
    build.build()
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, re.S)
    assert blocks, "the README holds no Python example"
    scope = {}
    torch.manual_seed(0)
    exec(blocks[0], scope)
    torch.cuda.synchronize()
    xs, outs = scope["xs"], scope["outs"]
    bits = [x.view(torch.int16).cpu().numpy().view(np.uint16) for x in xs]
    ref, _ = O.allreduce(bits, "fp8")                  # the last call wrote FP8 results into outs
    for o in outs:
        assert np.array_equal(o.view(torch.int16).cpu().numpy().view(np.uint16), ref[0])
    host = scope["host"]
    ref4, _ = O.allreduce(bits, "int4")
    for h in host:
        assert np.array_equal(h.view(torch.int16).numpy().view(np.uint16), ref4[0])
