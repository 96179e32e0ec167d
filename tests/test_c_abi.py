"""The C ABI from a plain C program (no GPU needed).

tests/c/abi_check.c includes include/sfp8.h as C99 (-Wall -Werror), takes the
address of every declared entry point, links against the built libsfp8.so
and calls the entry points that touch no device (layout sizes, status
strings, the host-only plan query for a 148-SM B200, argument validation).
"""
import os
import shutil
import subprocess

import pytest

from semi_structured_sparse_rowwise_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(tmp_path):
    lib = build.build()
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_check.c"),
           "-L", os.path.dirname(lib), "-l:" + os.path.basename(lib),
           "-Wl,-rpath," + os.path.dirname(lib), "-o", str(exe)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "abi ok", (r.returncode, r.stdout, r.stderr)
