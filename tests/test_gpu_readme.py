"""The README's usage examples run as written (all its python blocks, in order,
in one namespace) and leave no device-side error behind."""
import os
import re

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_examples_run():
    from paged_kv_cache_404_b200 import build
    build.build()
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, re.S)
    assert len(blocks) >= 5
    ns = {}
    for b in blocks:
        exec(compile(b, "README.md", "exec"), ns)
    torch.cuda.synchronize()
    assert torch.isfinite(ns["out"].float()).all() and torch.isfinite(ns["out1"].float()).all()
    assert torch.isfinite(ns["out3"].float()).all()
    assert ns["cached"] == (ns["L"] // 16) * 16       # every full block of the prompt was reused
    assert ns["bm"].is_swapped(ns["seq"]) is False
