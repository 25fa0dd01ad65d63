"""The CUDA library and the CPU oracle share no code, and the product path
has no CPU fallback.

  * no module of the package imports the oracle, and the oracle imports
    nothing of the package;
  * no CUDA source includes an oracle file and the oracle's C source includes
    neither the library's header nor its kernel headers;
  * bench.py touches the oracle only in its CPU-baseline and reference legs;
  * with libw4.so missing, the binding raises instead of computing anything.
"""
import ast
import glob
import os
import re

import numpy as np
import pytest

from conftest import ROOT

PKG = os.path.join(ROOT, "bit_gemm_quant_b200")
ORACLE = os.path.join(ROOT, "oracle")


def imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.level == 0 and node.module:
            names.add(node.module.split(".")[0])
    return names


def test_package_never_imports_the_oracle():
    for path in glob.glob(os.path.join(PKG, "*.py")):
        assert "oracle" not in imported_modules(path), path


def test_oracle_never_imports_the_package():
    for path in glob.glob(os.path.join(ORACLE, "*.py")):
        assert "bit_gemm_quant_b200" not in imported_modules(path), path


def test_sources_share_no_headers():
    for path in glob.glob(os.path.join(PKG, "csrc", "*")):
        for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', open(path).read()):
            assert "oracle" not in inc, (path, inc)
    for path in glob.glob(os.path.join(ORACLE, "*.c")) + glob.glob(os.path.join(ORACLE, "*.h")):
        for inc in re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', open(path).read()):
            assert inc not in ("w4.h", "common.cuh", "tc_ptx.cuh") and "csrc" not in inc, (path, inc)


def test_bench_uses_the_oracle_only_in_its_cpu_legs():
    path = os.path.join(ROOT, "bench.py")
    tree = ast.parse(open(path).read(), filename=path)
    allowed = ("cpu_baseline", "run_reference")
    for fn in [n for n in ast.walk(tree) if isinstance(n, ast.FunctionDef)]:
        for node in ast.walk(fn):
            mods = []
            if isinstance(node, ast.Import):
                mods = [a.name.split(".")[0] for a in node.names]
            elif isinstance(node, ast.ImportFrom) and node.module:
                mods = [node.module.split(".")[0]]
            if "oracle" in mods:
                assert fn.name.startswith(allowed), "bench.py imports the oracle in %s" % fn.name
    top = [n for n in tree.body if isinstance(n, (ast.Import, ast.ImportFrom))]
    for node in top:
        names = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
        assert not any(n.split(".")[0] == "oracle" for n in names)


def test_missing_library_raises(monkeypatch):
    import torch
    import bit_gemm_quant_b200 as w4
    monkeypatch.setattr(w4, "_LIB_PATH", os.path.join(ROOT, "no_such_dir", "libw4.so"))
    monkeypatch.setattr(w4, "_lib", None)
    # the raw entry points load the library first
    with pytest.raises(RuntimeError, match="not built"):
        w4.w4_quant_pack(None, 16, 256, 128, w4.SYM, None, None, None, None, None)
    with pytest.raises(RuntimeError, match="not built"):
        w4.w4_fp4_quant(None, 16, 256, w4.NVFP4, None, None, None)
    with pytest.raises(RuntimeError, match="not built"):
        w4.w4a16_workspace_bytes(32, 256, 256, 128)
    # the tensor helpers raise too (on a machine without CUDA already at the
    # stream lookup): nothing is computed on the host
    W = torch.zeros((16, 256), dtype=torch.bfloat16)
    for call in (lambda: w4.quant_pack(W, 128, w4.SYM), lambda: w4.fp4_quant(W, w4.NVFP4)):
        with pytest.raises(RuntimeError):
            call()
