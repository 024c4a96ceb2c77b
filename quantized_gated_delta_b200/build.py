"""Build libstepq.so (the C ABI in include/stepq.h) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libstepq.so")
SOURCES = ["stepq_decode.cu", "stepq_io.cu", "stepq_capi.cu", "stepq_alloc.cpp"]
HEADERS = ["stepq_device.cuh", "stepq_tile.cuh", "stepq_internal.h"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-O3", "-std=c++17",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart=static",
    "-Xptxas", "-v",
    "-I" + os.path.join(ROOT, "include"),
]
BUILD_LOG = os.path.join(HERE, "_build", "nvcc.log")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    files.append(os.path.join(ROOT, "include", "stepq.h"))
    files.append(os.path.abspath(__file__))
    return files


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


def build(force: bool = False, quiet: bool = True) -> str:
    """Compile the library if any input is newer than it; returns its path."""
    if not force and not stale():
        return LIB
    os.makedirs(os.path.dirname(BUILD_LOG), exist_ok=True)
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = [NVCC, *FLAGS, "-o", tmp, *[os.path.join(CSRC, f) for f in SOURCES]]
    proc = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    with open(BUILD_LOG, "w") as fh:
        fh.write(" ".join(cmd) + "\n" + proc.stdout + proc.stderr)
    if proc.returncode != 0:
        sys.stderr.write(proc.stdout + proc.stderr)
        raise RuntimeError("nvcc failed (log: %s)" % BUILD_LOG)
    os.replace(tmp, LIB)
    if not quiet:
        sys.stdout.write(proc.stderr)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, quiet=False)
    print(LIB)
