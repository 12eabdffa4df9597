"""include/fqa.h compiles as C99 and libfqa.so links into a plain C program,
which then exercises the calls that need no GPU (tests/c/abi_from_c.c)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB_DIR = os.path.join(ROOT, "quantized_fp8_attention_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_and_library_from_plain_c(tmp_path):
    from quantized_fp8_attention_b200 import build
    build.build()
    exe = tmp_path / "abi_from_c"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-L", LIB_DIR, "-lfqa",
                    f"-Wl,-rpath,{LIB_DIR}", "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "OK (0 failed)" in r.stdout
