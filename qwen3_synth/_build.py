"""Builds lib/libqwen3synth.so (host OpenMP + CUDA generators of the seeded inputs)
with nvcc for sm_100a; rebuilt only when the source or the flags changed."""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "synth.cu")
LIB = os.path.join(HERE, "lib")
TARGET = os.path.join(LIB, "libqwen3synth.so")
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-fopenmp",
         "-gencode", "arch=compute_100a,code=sm_100a"]


def build(verbose: bool = False, force: bool = False) -> str:
    os.makedirs(LIB, exist_ok=True)
    h = hashlib.sha256(open(SRC, "rb").read())
    h.update(" ".join(FLAGS).encode())
    stamp = TARGET + ".stamp"
    if not force and os.path.exists(TARGET) and os.path.exists(stamp) and open(stamp).read() == h.hexdigest():
        return TARGET
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    cmd = [nvcc, *FLAGS, "-shared", SRC, "-o", TARGET, "-lgomp"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {SRC}:\n{r.stderr}")
    with open(stamp, "w") as f:
        f.write(h.hexdigest())
    if verbose:
        print(f"built {TARGET}", file=sys.stderr)
    return TARGET


if __name__ == "__main__":
    print(build(verbose=True, force="--force" in sys.argv))
