"""build() must work in a fresh checkout, where libqf.so does not exist yet: the
package's __init__ loads the library, so the builder is loaded by file path and the
package is imported only after the build."""
import subprocess
import sys
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_loading_the_builder_imports_no_part_of_the_package():
    code = ("import sys, __graft_entry__ as g\n"
            "m = g._load_file('qf_build', 'fp4_fake_quant_b200', '_build.py')\n"
            "assert callable(m.build)\n"
            "bad = [k for k in sys.modules if k.startswith('fp4_fake_quant_b200')]\n"
            "assert not bad, bad\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
