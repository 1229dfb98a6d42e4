"""CPU checks of the separation between the product, the oracle and the input generators:
the library package never reaches the oracle, the oracle and the generators never reach the
library (and hold no CUDA or torch code), and the binding refuses to load without the built
CUDA library instead of falling back to anything else."""
import ast
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = "rank_kv_cache_lr_b200"


def _imports(path):
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom):
            if node.level == 0 and node.module:
                names.add(node.module.split(".")[0])
    return names


def _py_files(folder):
    for dirpath, _, files in os.walk(os.path.join(ROOT, folder)):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(dirpath, f)


def test_product_package_never_imports_the_oracle():
    for path in _py_files(PKG):
        bad = _imports(path) & {"oracle", "synth", "tests"}
        assert not bad, f"{path} imports {bad}"


def test_product_sources_never_include_oracle_code():
    csrc = os.path.join(ROOT, PKG, "csrc")
    for f in os.listdir(csrc):
        text = open(os.path.join(csrc, f)).read()
        for line in text.splitlines():
            if line.lstrip().startswith("#include"):
                assert "oracle" not in line and "synth" not in line, f"{f}: {line}"


@pytest.mark.parametrize("folder", ["oracle", "synth"])
def test_oracle_and_generators_stay_off_the_library(folder):
    allowed = {"numpy", "math", "dataclasses", "hashlib", "typing", "__future__", "itertools",
               "functools", "collections", "json", "os"}
    for path in _py_files(folder):
        names = _imports(path)
        assert PKG not in names and "torch" not in names and "ctypes" not in names, (path, names)
        assert names <= allowed | {"oracle", "synth"}, (path, names - allowed)
    if folder == "synth":
        for path in _py_files(folder):
            assert "oracle" not in _imports(path), path


def test_binding_refuses_to_load_without_the_library(tmp_path):
    """A copy of the package without `_lib/` must fail at import: no CPU path exists."""
    dst = tmp_path / PKG
    shutil.copytree(os.path.join(ROOT, PKG), dst,
                    ignore=shutil.ignore_patterns("_lib", "__pycache__", "csrc"))
    code = f"import sys; sys.path.insert(0, {str(tmp_path)!r}); import {PKG}"
    res = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert res.returncode != 0
    assert "CUDA library not built" in res.stderr
