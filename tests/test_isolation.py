"""The oracle and the product path stay apart, and the product path has no fallback.

Checked on the host, without a GPU:
- nothing in the package (Python binding, CUDA sources, headers) or in include/
  imports, links or names the oracle;
- nothing in oracle/ includes or imports the package's sources;
- bench.py loads the oracle only inside OracleStep, which serves the
  cpu_baseline and reference legs;
- with the CUDA library missing, the binding's first call raises instead of
  computing anything another way.
"""
import ast
import os
import re

import pytest

from compressed_domain_attention_b200 import tq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "compressed_domain_attention_b200")
SOURCE_EXT = (".py", ".cu", ".cuh", ".h", ".cpp", ".c")


def sources(top):
    for d, _, files in os.walk(top):
        if "__pycache__" in d:
            continue
        for f in files:
            if f.endswith(SOURCE_EXT):
                yield os.path.join(d, f)


def test_product_sources_never_name_the_oracle():
    pat = re.compile(r"\bimport\s+oracle\b|\bfrom\s+oracle\b|tq_oracle|libtq_oracle|oracle/")
    hits = []
    for top in (PKG, os.path.join(ROOT, "include")):
        for path in sources(top):
            for i, line in enumerate(open(path, encoding="utf-8"), 1):
                if pat.search(line):
                    hits.append(f"{os.path.relpath(path, ROOT)}:{i}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_oracle_never_uses_the_product_sources():
    pat = re.compile(r"^\s*(import|from)\s+compressed_domain_attention_b200|#\s*include\s*[<\"][^>\"]*"
                     r"(tq_device|tq_kernels|tq\.h)|libtq_b200|csrc/")
    hits = []
    for path in sources(os.path.join(ROOT, "oracle")):
        for i, line in enumerate(open(path, encoding="utf-8"), 1):
            if pat.search(line):
                hits.append(f"{os.path.relpath(path, ROOT)}:{i}: {line.strip()}")
    assert not hits, "\n".join(hits)


def test_bench_loads_the_oracle_only_in_its_oracle_leg():
    tree = ast.parse(open(os.path.join(ROOT, "bench.py"), encoding="utf-8").read())
    where = []

    def visit(node, scope):
        for child in ast.iter_child_nodes(node):
            inner = scope
            if isinstance(child, (ast.FunctionDef, ast.ClassDef)):
                inner = scope + [child.name]
            if isinstance(child, ast.Import) and any(a.name.split(".")[0] == "oracle" for a in child.names):
                where.append(inner)
            if isinstance(child, ast.ImportFrom) and (child.module or "").split(".")[0] == "oracle":
                where.append(inner)
            visit(child, inner)

    visit(tree, [])
    assert where, "bench.py no longer times the oracle"
    assert all(s and s[0] == "OracleStep" for s in where), where


def test_missing_library_raises_on_first_call(monkeypatch, tmp_path):
    monkeypatch.setattr(tq, "LIB_PATH", str(tmp_path / "libtq_b200.so"))
    monkeypatch.setattr(tq, "_LIB", None)
    with pytest.raises(ImportError, match="no CPU fallback"):
        tq.tq_cache_layout(1, 16, 1, 1, 128)
