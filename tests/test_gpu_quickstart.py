"""The quick-start example (examples/quickstart.py) runs as written, in a scratch
directory, and writes its checkpoint shard."""
import os
import runpy
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_quickstart_example(tmp_path, monkeypatch):
    monkeypatch.chdir(tmp_path)
    monkeypatch.setattr(sys, "path", [ROOT] + sys.path)
    runpy.run_path(os.path.join(ROOT, "examples", "quickstart.py"), run_name="quickstart")
    assert (tmp_path / "model-00001.safetensors").stat().st_size > 0
