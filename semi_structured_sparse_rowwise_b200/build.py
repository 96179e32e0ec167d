"""Builds libsfp8.so in-tree with nvcc for sm_100a.

    python -m semi_structured_sparse_rowwise_b200.build [--verbose]

The library is one translation unit (csrc/sfp8_api.cu including the kernel
headers), linked against the static CUDA runtime so that it needs nothing
from the Python environment.  The driver API entry it uses
(cuTensorMapEncodeTiled) is looked up at run time through the runtime.
"""

import os
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
CSRC = os.path.join(PKG_DIR, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libsfp8.so"
LIB_PATH = os.path.join(PKG_DIR, LIB_NAME)

SOURCES = ["sfp8_api.cu"]


def nvcc_path():
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found; set NVCC or install the CUDA toolkit")
    return cand


def _inputs():
    headers = sorted(f for f in os.listdir(CSRC) if f.endswith(".cuh"))
    files = [os.path.join(CSRC, f) for f in SOURCES + headers]
    files.append(os.path.join(INCLUDE, "sfp8.h"))
    files.append(os.path.abspath(__file__))
    return files


def up_to_date():
    if not os.path.exists(LIB_PATH):
        return False
    t = os.path.getmtime(LIB_PATH)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(verbose=False, force=False, extra_flags=()):
    """Compile libsfp8.so next to this file; returns its path."""
    if not force and up_to_date():
        return LIB_PATH
    tmp = LIB_PATH + ".tmp"
    cmd = [
        nvcc_path(), "-O3", "-std=c++17",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-lineinfo", "-Xcompiler", "-fPIC,-O3", "-shared",
        "-cudart", "static",
        "-I", INCLUDE, "-I", CSRC,
        "-o", tmp,
    ]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += list(extra_flags)
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stdout.write(res.stdout)
        sys.stderr.write(res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building %s (exit %d)" % (LIB_NAME, res.returncode))
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force="--force" in sys.argv)
    print(LIB_PATH)
