"""The product / oracle boundary, on CPU: the library and its binding never reach the oracle
(and the oracle never reaches them), bench.py and the entry module load the oracle only in the
legs that time or check against it (and to compile it), and the binding fails loudly when
libtg.so is missing instead of falling back to anything."""
import ast
import os
import re

import pytest

import non_uniform_paged_flash_b200 as tg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "non_uniform_paged_flash_b200")
ORACLE = os.path.join(ROOT, "oracle")


def _sources(top, exts):
    for d, _, files in os.walk(top):
        for f in files:
            if f.endswith(exts):
                yield os.path.join(d, f)


def test_product_never_names_the_oracle():
    pat = re.compile(r"\boracle\b|_liboracle|tg_oracle|\bor_[a-z0-9_]+\(")
    hits = []
    for path in _sources(PKG, (".py", ".cu", ".cpp", ".h")):
        with open(path, encoding="utf-8") as f:
            for n, line in enumerate(f, 1):
                if pat.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{n}: {line.strip()}")
    with open(os.path.join(ROOT, "include", "tg.h"), encoding="utf-8") as f:
        hits += [f"include/tg.h:{n}" for n, line in enumerate(f, 1) if pat.search(line)]
    assert not hits, "\n".join(hits)


def test_oracle_never_names_the_product():
    pat = re.compile(r"^\s*(import|from)\s+non_uniform_paged_flash_b200|libtg\.so|#\s*include\s*[<\"]tg|"
                     r"csrc/|\btg_[a-z0-9_]+\(")
    hits = []
    for path in _sources(ORACLE, (".py", ".c", ".h")):
        with open(path, encoding="utf-8") as f:
            for n, line in enumerate(f, 1):
                if pat.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{n}: {line.strip()}")
    assert not hits, "\n".join(hits)


def _oracle_imports(path):
    """(function name or '<module>', line) of every import of the oracle package."""
    with open(path, encoding="utf-8") as f:
        tree = ast.parse(f.read())
    found = []

    def visit(node, where):
        for child in ast.iter_child_nodes(node):
            inner = child.name if isinstance(child, (ast.FunctionDef, ast.AsyncFunctionDef)) else where
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                found.append((where, child.lineno))
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                found.append((where, child.lineno))
            visit(child, inner)

    visit(tree, "<module>")
    return found


@pytest.mark.parametrize("name,allowed", [("bench.py", {"cpu_baseline", "run_reference"}),
                                          ("__graft_entry__.py", {"build", "smoke"})])
def test_oracle_loaded_only_by_its_legs(name, allowed):
    found = _oracle_imports(os.path.join(ROOT, name))
    assert found, f"{name} no longer loads the oracle anywhere: update this test"
    assert {w for w, _ in found} <= allowed, found


def test_binding_fails_loudly_without_the_library(monkeypatch):
    monkeypatch.setattr(tg, "LIB_PATH", os.path.join(ROOT, "no_such_dir", "libtg.so"))
    monkeypatch.setattr(tg, "_L", None)
    with pytest.raises(ImportError):
        tg.load()
    with pytest.raises(ImportError):
        tg.tg_splitzip_workspace_bytes(16)
