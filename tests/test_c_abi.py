"""The C ABI from plain C: tests/c_abi_check.c includes include/q8.h as a C99 translation
unit (warnings as errors), links against libq8.so and calls every entry point that can be
decided on the host, checking the documented status codes.  No device work."""
import os
import shutil
import subprocess

import pytest

import int8_quantized_linear_q8_b200 as q8
from int8_quantized_linear_q8_b200 import build as q8build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c99_caller(tmp_path):
    q8build.build()
    libdir = os.path.dirname(q8.LIB_PATH)
    exe = str(tmp_path / "c_abi_check")
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "c_abi_check.c"),
                           "-L", libdir, "-lq8", "-Wl,-rpath," + libdir, "-o", exe])
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "failures: 0" in out.stdout
