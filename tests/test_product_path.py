"""The product path is the CUDA library alone: no CPU fallback, no route through the oracle."""
import ast
import os

import pytest
import torch

import thinned_softmax_attention_b200 as tab

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "thinned_softmax_attention_b200")


def _imported_modules(path):
    tree = ast.parse(open(path).read(), path)
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            for a in node.names:
                yield a.name
        elif isinstance(node, ast.ImportFrom):
            yield node.module or ""


def test_package_never_imports_the_oracle():
    files = [os.path.join(d, f) for d, _, fs in os.walk(PKG) for f in fs if f.endswith(".py")]
    files.append(os.path.join(ROOT, "workloads.py"))
    assert files
    for path in files:
        for mod in _imported_modules(path):
            assert not mod.split(".")[0] == "oracle", f"{path} imports {mod}"


def test_missing_library_raises(monkeypatch):
    monkeypatch.setattr(tab, "_lib", None)
    monkeypatch.setattr(tab, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libthin_attn.so"))
    with pytest.raises(ImportError, match="is missing"):
        tab.lib()
    with pytest.raises(ImportError):
        tab.ThinAttention(B=1, T=16, S=16, H=1, E=64, D=64, dtype=torch.bfloat16)
