"""The CUDA path and the oracle share no code, and the product has no CPU
fallback: no product module imports the oracle, neither side includes the other's
sources, nothing reads the reference pages at run time, and a missing library
raises instead of computing elsewhere.  No GPU."""
import ast
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "test_sequence_modeling_b200")
CSRC = os.path.join(PKG, "csrc")


def _product_modules():
    return [os.path.join(PKG, f) for f in sorted(os.listdir(PKG)) if f.endswith(".py")]


def test_product_modules_do_not_import_the_oracle():
    for path in _product_modules():
        tree = ast.parse(open(path).read(), path)
        for node in ast.walk(tree):
            names = []
            if isinstance(node, ast.Import):
                names = [a.name for a in node.names]
            elif isinstance(node, ast.ImportFrom):
                names = [node.module or ""]
            for n in names:
                assert not n.split(".")[0] == "oracle", f"{path} imports {n}"


def test_cuda_sources_and_oracle_share_no_includes():
    cuda = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    for path in cuda:
        for inc in re.findall(r'#include\s+[<"]([^>"]+)[>"]', open(path).read()):
            assert "oracle" not in inc, (path, inc)
    oracle_c = os.path.join(ROOT, "oracle", "ttt_oracle.c")
    for inc in re.findall(r'#include\s+[<"]([^>"]+)[>"]', open(oracle_c).read()):
        assert not inc.startswith(("cuda", "ttt.h")) and not inc.endswith(".cuh"), inc


def test_nothing_reads_files_outside_the_repository():
    """No product file, bench.py or the entry points names an absolute filesystem
    path (a quoted string starting with '/'): everything they read lives in the
    repository, so nothing reads the reference pages or any other outside file."""
    files = _product_modules() + [os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py")]
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    files += [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))]
    pattern = re.compile(r"""["'](/[A-Za-z_][^"'\n]*)["']""")
    for path in files:
        found = pattern.findall(open(path).read())
        assert not found, (path, found)


def test_missing_library_raises():
    from test_sequence_modeling_b200 import _lib
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load(os.path.join(ROOT, "no_such_libttt.so"))
