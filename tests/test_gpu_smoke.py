"""The entry point's smoke() (one small block forward on cuda:0, checked
against the oracle) runs as part of the GPU suite."""
import importlib.util
import os

import pytest

pytestmark = pytest.mark.gpu


def test_graft_entry_smoke_runs():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("graft_entry", os.path.join(root, "__graft_entry__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.smoke()
