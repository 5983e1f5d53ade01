"""Build libalhr.so in-tree with nvcc for sm_100a.

    python -m tree_routed_sparse_b200.build [--force] [--verbose-ptxas]

The library is rebuilt when the hash of its sources (csrc/*, include/alhr.h, this file)
changes; the hash is kept beside the library.
"""
from __future__ import annotations

import glob
import hashlib
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIB_DIR, "libalhr.so")
STAMP = LIB + ".srchash"
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")

FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "--expt-relaxed-constexpr",
]


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(PKG, "csrc", "*.cu")))


def _hash() -> str:
    h = hashlib.sha1()
    files = sorted(glob.glob(os.path.join(PKG, "csrc", "*"))) + [
        os.path.join(ROOT, "include", "alhr.h"), os.path.abspath(__file__)]
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    h.update(" ".join(FLAGS).encode())
    return h.hexdigest()


HEADERS = ["alhr_device.cuh", "internal.h", "tree_layout.h", "query_common.cuh"]


def code_only(text: str) -> str:
    """C/C++/CUDA source without its comments and blank lines (the sources hold no string
    literal with a comment marker)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def kernel_hash(source: str) -> str:
    """Hash of the code (comments and blank lines left out) of one csrc/*.cu file, the headers
    every source includes, and the flags: it identifies the kernels defined in that file, so a
    stored profiler record of one kernel stays valid while only other files or comments
    change."""
    h = hashlib.sha1()
    files = [os.path.join(PKG, "csrc", source)] + [
        os.path.join(PKG, "csrc", x) for x in HEADERS] + [os.path.join(ROOT, "include", "alhr.h")]
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    h.update(" ".join(FLAGS).encode())
    return h.hexdigest()


def is_current() -> bool:
    if not os.path.exists(LIB) or not os.path.exists(STAMP):
        return False
    with open(STAMP) as f:
        return f.read().strip() == _hash()


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not ptxas_verbose and is_current():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"), "-o", tmp, *sources()]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(_hash())
    return LIB


if __name__ == "__main__":
    path = build(force="--force" in sys.argv, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(path)
