"""There is no CPU or library fallback: without the compiled library the
package refuses to import, and every compute entry point refuses CPU tensors."""
import os
import shutil
import subprocess
import sys

from conftest import ROOT


def test_package_without_library_refuses_to_import(tmp_path):
    pkg = os.path.join(ROOT, "bit_nf4_quantized_05_b200")
    dst = tmp_path / "bit_nf4_quantized_05_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("_lib", "__pycache__", "csrc"))
    r = subprocess.run([sys.executable, "-c", "import bit_nf4_quantized_05_b200"],
                       capture_output=True, text=True, cwd=str(tmp_path), timeout=300,
                       env=dict(os.environ, PYTHONPATH=str(tmp_path)))
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "no fallback" in r.stderr
