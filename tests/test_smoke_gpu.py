"""The build entry's smoke check on the GPU (one small call checked against the oracle)."""
import importlib.util
import os

import pytest

from gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def test_build_entry_smoke():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("_entry", os.path.join(root, "__graft_entry__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.smoke()
