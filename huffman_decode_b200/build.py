"""Builds the DF11 shared library (host codec + sm_100a decode kernel) in-tree.

    python -m huffman_decode_b200.build        # or build() from Python

Output: huffman_decode_b200/_lib/libdf11.so, exporting the C ABI declared in
include/df11.h, and libdf11_checked.so, the same library built with
-DDF11_CHECKED (run-time bound checks in the decode kernel; the binding loads
it when DF11_CHECKED=1).  nvcc cross-compiles for sm_100a without a GPU.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
INCLUDE = os.path.join(ROOT, "include")
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "_lib")
LIB_PATH = os.path.join(LIB_DIR, "libdf11.so")
CHECKED_LIB_PATH = os.path.join(LIB_DIR, "libdf11_checked.so")

SOURCES = [os.path.join(CSRC, f) for f in ("df11_host.cpp", "df11_decode.cu", "df11_encode.cu", "df11_pipeline.cpp", "df11_crc.cu",
                                                 "df11_io.cpp")]
HEADERS = [os.path.join(INCLUDE, "df11.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O3,-pthread",
    "-shared",
]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def is_stale(path: str = LIB_PATH) -> bool:
    if not os.path.exists(path):
        return True
    built = os.path.getmtime(path)
    return any(os.path.getmtime(f) > built for f in SOURCES + HEADERS + [__file__])


def _compile(path: str, extra, verbose: bool) -> None:
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = path + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *NVCC_FLAGS, *extra, f"-I{INCLUDE}", *SOURCES, "-o", tmp]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, path)


def build(force: bool = False, verbose: bool = False, checked: bool = False) -> str:
    """Compile the library (checked=True: the bound-checked one) if a source
    is newer than it (or force); returns its path."""
    path = CHECKED_LIB_PATH if checked else LIB_PATH
    if force or is_stale(path):
        _compile(path, ["-DDF11_CHECKED"] if checked else [], verbose)
    return path


def build_all(force: bool = False, verbose: bool = False) -> list:
    return [build(force, verbose, checked=False), build(force, verbose, checked=True)]


if __name__ == "__main__":
    print(build_all(force="--force" in sys.argv, verbose=True))
