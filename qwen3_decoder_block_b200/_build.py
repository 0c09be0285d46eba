"""Builds the in-tree shared libraries with nvcc for sm_100a.

    lib/libqwen3blk.so    the decoder-block library (C ABI in include/qwen3blk.h)

Each translation unit is compiled to an object in parallel, then linked; a
library is rebuilt only when a source, header or flag changed.
"""
from __future__ import annotations

import concurrent.futures as cf
import hashlib
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "lib")
OBJ = os.path.join(LIB, "obj")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
NVCC_FLAGS = ["-O3", "-std=c++17", "-lineinfo", "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC",
              "-Xcompiler", "-fopenmp", "-Xptxas", "-v"] + ARCH

LIBRARIES = {
    "libqwen3blk.so": ["api.cu", "gemm.cu", "gemm_skinny.cu", "elementwise.cu", "attention.cu", "moe.cu"],
}
HEADERS = ["common.cuh", "internal.h"]


def _nvcc() -> str:
    p = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(p):
        raise RuntimeError("nvcc not found")
    return p


def _digest(paths, extra) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(p, "rb") as f:
            h.update(f.read())
    h.update(" ".join(extra).encode())
    return h.hexdigest()


def _compile(src: str, obj: str) -> tuple[str, str]:
    cmd = [_nvcc(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"), "-c", src, "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    return src, r.stderr


def build(verbose: bool = False, force: bool = False) -> dict:
    os.makedirs(OBJ, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(ROOT, "include", "qwen3blk.h")]
    out = {}
    for lib, srcs in LIBRARIES.items():
        paths = [os.path.join(CSRC, s) for s in srcs]
        stamp = os.path.join(LIB, lib + ".stamp")
        target = os.path.join(LIB, lib)
        dig = _digest(paths + headers, NVCC_FLAGS)
        if not force and os.path.exists(target) and os.path.exists(stamp) and open(stamp).read() == dig:
            out[lib] = target
            continue
        objs = [os.path.join(OBJ, os.path.splitext(s)[0] + ".o") for s in srcs]
        logs = {}
        with cf.ThreadPoolExecutor(max_workers=min(8, len(srcs))) as ex:
            for src, log in ex.map(lambda a: _compile(*a), zip(paths, objs)):
                logs[src] = log
        link = [_nvcc(), "-shared", *ARCH, "-Xcompiler", "-fopenmp", "-o", target, *objs, "-lgomp"]
        r = subprocess.run(link, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"link of {lib} failed:\n{r.stderr}")
        with open(os.path.join(LIB, lib + ".ptxas.log"), "w") as f:
            for src, log in logs.items():
                f.write(f"== {os.path.basename(src)}\n{log}\n")
        with open(stamp, "w") as f:
            f.write(dig)
        if verbose:
            print(f"built {target}", file=sys.stderr)
        out[lib] = target
    return out


if __name__ == "__main__":
    for k, v in build(verbose=True, force="--force" in sys.argv).items():
        print(k, v)
