"""The C ABI used from plain C: tests/c/abi_from_c.c is compiled with gcc
against include/hq.h, linked to libhq.so and run on the host (packing,
sizes and argument errors; no GPU needed)."""

import os
import shutil
import subprocess
import tempfile

import pytest

from quantized_gemm_bit_b200 import hq
from quantized_gemm_bit_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_abi():
    build()
    libdir = os.path.dirname(hq.LIB_PATH)
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "abi_from_c")
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                        os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-o", exe, "-L", libdir, "-lhq",
                        "-Wl,-rpath," + libdir], check=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
        assert r.returncode == 0, r.stderr
        assert r.stdout.strip() == "ok"
