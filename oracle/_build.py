"""Builds lib/libqwen3ref.so, the fp64 C++ oracle (test infrastructure), with g++ and
OpenMP; rebuilt only when the source or the flags changed."""
from __future__ import annotations

import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qwen3_ref.cpp")
LIB = os.path.join(HERE, "lib")
TARGET = os.path.join(LIB, "libqwen3ref.so")
FLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-Wall", "-Wextra"]


def build(verbose: bool = False, force: bool = False) -> str:
    os.makedirs(LIB, exist_ok=True)
    h = hashlib.sha256(open(SRC, "rb").read())
    h.update(" ".join(FLAGS).encode())
    stamp = TARGET + ".stamp"
    if not force and os.path.exists(TARGET) and os.path.exists(stamp) and open(stamp).read() == h.hexdigest():
        return TARGET
    cxx = shutil.which("g++") or "g++"
    r = subprocess.run([cxx, *FLAGS, SRC, "-o", TARGET], capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"g++ failed for {SRC}:\n{r.stderr}")
    with open(stamp, "w") as f:
        f.write(h.hexdigest())
    if verbose:
        print(f"built {TARGET}", file=sys.stderr)
    return TARGET


if __name__ == "__main__":
    print(build(verbose=True, force="--force" in sys.argv))
