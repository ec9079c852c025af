"""The C ABI used from a C program (gcc, include/dsa.h, libdsa.so): host-side entry points
and argument checks, no GPU."""

import os
import shutil
import subprocess

import pytest

from long_context_dsa_b200 import dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_against_the_header(tmp_path):
    if not os.path.exists(dsa.LIB_PATH):
        import long_context_dsa_b200.build as b
        b.build()
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(dsa.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_check.c"), "-L", libdir, "-ldsa",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
