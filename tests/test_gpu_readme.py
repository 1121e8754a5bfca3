"""The README's Python example runs as written (in a scratch directory)."""
import os

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_python_example(tmp_path, monkeypatch):
    text = open(os.path.join(ROOT, "README.md")).read()
    start = text.index("```python\n") + len("```python\n")
    code = text[start:text.index("```", start)]
    monkeypatch.chdir(tmp_path)
    exec(compile(code, "README.md", "exec"), {"__name__": "readme_example"})
    assert (tmp_path / "model-00001.safetensors").stat().st_size > 0
