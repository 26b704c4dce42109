"""CPU checks of the separation between the product and its test oracle.

- The package (binding, data-parallel helpers, build script) never imports the
  oracle, and the oracle never imports the package or reads its sources.
- The library sources share no file with the oracle.
- Without the built library the product fails loudly instead of falling back.
"""
from __future__ import annotations

import ast
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "bit_nf4_quantized_absmax_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _imports(path: str) -> set[str]:
    tree = ast.parse(open(path).read(), filename=path)
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _py_files(d: str):
    for base, _, files in os.walk(d):
        for f in files:
            if f.endswith(".py"):
                yield os.path.join(base, f)


def test_package_does_not_import_the_oracle():
    for f in _py_files(PKG):
        assert "oracle" not in _imports(f), f


def test_oracle_does_not_import_the_package():
    for f in _py_files(ORACLE):
        imp = _imports(f)
        assert "bit_nf4_quantized_absmax_b200" not in imp, f
        assert "csrc" not in open(f).read(), f


def test_no_source_file_is_shared():
    lib = {f for f in os.listdir(os.path.join(PKG, "csrc"))}
    orc = {f for f in os.listdir(ORACLE)}
    assert not (lib & orc - {"__pycache__"})


def test_missing_library_fails_loudly(monkeypatch):
    from bit_nf4_quantized_absmax_b200 import binding as b
    monkeypatch.setattr(b, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        b.load_library(os.path.join(ROOT, "no_such_dir", "libqlora_b200.so"))
