"""Builds libhash_scored_top.so in-tree (nvcc, sm_100a).

Run as ``python -m hash_scored_top_b200.build``. The library is the whole
compute path; the Python package only marshals arguments into it.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_NAME = "libhash_scored_top.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
SOURCES = ["csrc/api.cu"]
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
]


def _inputs():
    out = [os.path.join(HERE, s) for s in SOURCES]
    csrc = os.path.join(HERE, "csrc")
    out += [os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cuh", ".cu", ".h"))]
    out.append(os.path.join(os.path.dirname(HERE), "include", "hash_scored_top.h"))
    return out


def up_to_date() -> bool:
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library if any source is newer than it. Returns its path."""
    if not force and up_to_date():
        return LIB_PATH
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB_PATH + ".tmp"
    cmd = [nvcc, *NVCC_FLAGS, "-o", tmp, *[os.path.join(HERE, s) for s in SOURCES]]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True, cwd=HERE)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
