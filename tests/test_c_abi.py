"""The header compiles as strict C99 and a plain C program links and calls the
library without Python (argument checks only, so no GPU is needed)."""
import os
import shutil
import subprocess

import pytest

from conftest import ROOT, build_library


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_caller(tmp_path):
    lib = build_library()
    libdir = os.path.dirname(lib)
    exe = tmp_path / "probe"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                         "-I" + os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_probe.c"),
                         "-L" + libdir, "-lqlora_nf4", "-Wl,-rpath," + libdir, "-o", str(exe)],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stderr
