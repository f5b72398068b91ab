"""The oracle and the CUDA path share no code, and the library has no CPU fallback.

Checked on the sources: nothing in the package imports or names the oracle, the oracle imports
nothing of the package, and the input generator (the one module both sides use) holds no import
of either.  The binding raises when libpoetx.so is missing instead of computing anything itself.
"""
import ast
import os
import re

import pytest

import orthogonal_equivalence_cnp_b200 as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "orthogonal_equivalence_cnp_b200")


def _imports(path):
    tree = ast.parse(open(path).read())
    names = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            names.update(a.name.split(".")[0] for a in node.names)
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            names.add(node.module.split(".")[0])
    return names


def _files(folder, exts):
    for dirpath, _, files in os.walk(folder):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(dirpath, f)


def test_package_never_touches_the_oracle():
    for path in _files(PKG, (".py",)):
        assert "oracle" not in _imports(path), path
        assert not re.search(r"\boracle\b|poetx_ref", open(path).read()), path
    for path in _files(os.path.join(PKG, "csrc"), (".cu", ".cuh", ".h")):
        assert "poetx_ref" not in open(path).read(), path


def test_oracle_never_touches_the_package():
    for path in _files(os.path.join(ROOT, "oracle"), (".py",)):
        imps = _imports(path)
        assert "orthogonal_equivalence_cnp_b200" not in imps and "torch" not in imps, path
        assert "libpoetx" not in open(path).read(), path


def test_input_generator_imports_neither_side():
    imps = _imports(os.path.join(ROOT, "poetx_inputs.py"))
    assert not imps & {"oracle", "orthogonal_equivalence_cnp_b200", "torch"}, imps


def test_missing_library_raises(monkeypatch, tmp_path):
    monkeypatch.setattr(P, "_lib", None)
    monkeypatch.setattr(P, "library_path", lambda: str(tmp_path / "libpoetx.so"))
    with pytest.raises(RuntimeError, match="missing"):
        P.lib()
