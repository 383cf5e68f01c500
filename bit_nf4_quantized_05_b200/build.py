"""Build the sm_100a CUDA library in-tree: bit_nf4_quantized_05_b200/_lib/libqlora_nf4.so."""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC_DIR = os.path.join(HERE, "csrc")
MAIN = os.path.join(SRC_DIR, "qlora_nf4.cu")
OUT_DIR = os.path.join(HERE, "_lib")
LIB = os.path.join(OUT_DIR, "libqlora_nf4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "qlora_nf4.h")

NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
    "-Xptxas", "-v",
]


def _sources():
    out = [HEADER]
    for f in sorted(os.listdir(SRC_DIR)):
        if f.endswith((".cu", ".cuh")):
            out.append(os.path.join(SRC_DIR, f))
    return out


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if it is missing or older than any source; return its path."""
    if not force and os.path.exists(LIB):
        t = os.path.getmtime(LIB)
        if all(os.path.getmtime(s) <= t for s in _sources()):
            return LIB
    os.makedirs(OUT_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, MAIN, "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libqlora_nf4.so")
    if verbose:
        sys.stderr.write(res.stderr)
    with open(os.path.join(OUT_DIR, "ptxas.txt"), "w") as f:
        f.write(res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
