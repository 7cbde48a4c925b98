"""The oracle and the CUDA path share no code, and the product path never reaches the oracle
(CPU only, by reading the sources).

- oracle/ imports neither the package nor synth, and its C file includes only the C library;
- the package (its Python and its CUDA sources) never names the oracle, so no call, include or
  load of it can exist there;
- synth/ (the seeded generators both sides use) imports neither side.
"""
import ast
import glob
import os
import re

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "gemm_dequant_gemv_q8_b200"


def imported_modules(path):
    tree = ast.parse(open(path).read(), filename=path)
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            mods.add(node.module.split(".")[0])
    return mods


def test_oracle_imports_neither_the_package_nor_synth():
    for path in glob.glob(os.path.join(ROOT, "oracle", "*.py")):
        mods = imported_modules(path)
        assert PKG not in mods and "synth" not in mods, (path, mods)


def test_oracle_c_includes_only_the_c_library():
    src = open(os.path.join(ROOT, "oracle", "oracle.c")).read()
    incs = re.findall(r'#\s*include\s*[<"]([^>"]+)[>"]', src)
    assert incs and all(i in {"math.h", "stdint.h", "stdlib.h", "string.h", "stdio.h"} for i in incs), incs


def test_package_never_names_the_oracle():
    files = glob.glob(os.path.join(ROOT, PKG, "*.py")) + glob.glob(os.path.join(ROOT, PKG, "csrc", "*"))
    files += glob.glob(os.path.join(ROOT, "include", "*.h"))
    assert files
    for path in files:
        text = open(path, errors="replace").read()
        assert not re.search(r"\boracle\b|liboracle|qo_[a-z]", text), path
    for path in glob.glob(os.path.join(ROOT, PKG, "*.py")):
        assert "oracle" not in imported_modules(path), path


def test_synth_imports_neither_side():
    mods = imported_modules(os.path.join(ROOT, "synth", "__init__.py"))
    assert PKG not in mods and "oracle" not in mods, mods
