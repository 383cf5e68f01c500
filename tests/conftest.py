import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def build_library() -> str:
    """Compile the CUDA library if needed (nvcc only, no GPU). The build script is
    loaded by path because importing the package itself needs the built library."""
    path = os.path.join(ROOT, "bit_nf4_quantized_05_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_qlora_nf4_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


def read_golden_kv(name: str) -> dict:
    """key = value lines of a golden fixture (comments start with '#')."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split("=", 1)
            out[k.strip()] = v.strip()
    return out


def read_golden_lines(name: str) -> list:
    with open(os.path.join(GOLDEN, name)) as f:
        return [l.strip() for l in f if l.strip() and not l.startswith("#")]


def pytest_sessionstart(session):
    # The package refuses to import without its compiled library, so compile it
    # (a no-op when it is newer than every source) before any test module loads.
    build_library()
