"""The product path never reaches the oracle and has no fallback: no module or source of the
package imports or names the oracle, and the binding raises when the library is missing."""
import ast
import os

import pytest

from conditional_sparse_attention_b200 import _lib

PKG = os.path.dirname(_lib.__file__)


def _package_files(exts):
    for root, _, files in os.walk(PKG):
        if "_build" in root or "lib" == os.path.basename(root):
            continue
        for f in files:
            if f.endswith(exts):
                yield os.path.join(root, f)


def test_no_package_module_imports_the_oracle():
    for path in _package_files((".py",)):
        tree = ast.parse(open(path).read(), path)
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                assert not any(a.name.split(".")[0] == "oracle" for a in node.names), path
            elif isinstance(node, ast.ImportFrom):
                assert (node.module or "").split(".")[0] != "oracle", path


def test_no_cuda_source_names_the_oracle():
    for path in _package_files((".cu", ".cuh", ".h")):
        assert "oracle" not in open(path).read().lower(), path


def test_binding_raises_without_the_library(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", os.path.join(PKG, "no_such_library.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        _lib.load()
