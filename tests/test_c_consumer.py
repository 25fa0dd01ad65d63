"""The C ABI from C: include/w4.h compiles as strict C99 with every warning
an error, and a C program linked against libw4.so runs the host-side paths
(tests/c/abi_consumer.c) on a machine without a GPU."""
import os
import shutil
import subprocess

import pytest

from conftest import ROOT


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_library(tmp_path):
    from bit_gemm_quant_b200 import build
    build.build()
    pkg = os.path.join(ROOT, "bit_gemm_quant_b200")
    exe = str(tmp_path / "abi_consumer")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
           "-o", exe, "-L", pkg, "-l:libw4.so", "-Wl,-rpath," + pkg]
    out = subprocess.run(cmd, capture_output=True, text=True)
    assert out.returncode == 0, out.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr + run.stdout
    assert "all checks held" in run.stdout
