"""The C ABI from plain C: tests/c/abi_client.c compiles with gcc against
include/engram.h alone (no CUDA or torch headers), links libengram.so and
runs its host-side calls (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

from hashed_gram_conditional_hash_b200 import _lib as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is not installed")
def test_plain_c_client_builds_links_and_runs(tmp_path):
    libdir = os.path.dirname(L.LIB_PATH)
    exe = str(tmp_path / "abi_client")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_client.c"), "-o", exe, "-L", libdir,
                    "-l:libengram.so", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "FAIL" not in out.stdout and out.stdout.count(" ok") == 8
