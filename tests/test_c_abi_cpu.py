"""The boundary is a C ABI: a C99 program that includes only include/nvfp4rac.h compiles with
-Wall -Werror, links against the shared library and gets the documented host-side results."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_caller(tmp_path):
    from nvfp4_w4a4_moe_02_b200 import build_lib

    build_lib.build()
    libdir = os.path.join(ROOT, "nvfp4_w4a4_moe_02_b200")
    exe = tmp_path / "abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-L", libdir, "-lnvfp4rac",
           "-Wl,-rpath," + libdir, "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c abi ok" in r.stdout, r.stdout + r.stderr
