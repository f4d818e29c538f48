"""The C ABI from C: tests/c_abi_check.c includes include/dspark.h as C99 (with
-Wall -Wextra -Werror -pedantic), links libdspark.so and checks the host-side
paths that need no GPU."""
import os
import shutil
import subprocess

import pytest

from speculative_decoding_draft_sample_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "speculative_decoding_draft_sample_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs a C compiler")
def test_c_caller(tmp_path):
    build.build()
    exe = str(tmp_path / "c_abi_check")
    cc = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
          os.path.join(ROOT, "tests", "c_abi_check.c"), "-I", os.path.join(ROOT, "include"),
          "-L", PKG, "-ldspark", "-Wl,-rpath," + PKG, "-o", exe]
    out = subprocess.run(cc, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and "c abi: ok" in run.stdout, run.stdout + run.stderr
