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


def test_nothing_reads_the_reference_pages():
    """No product file, bench.py or the entry points names the location of the
    reference pages (taken from the workload description beside the repository)."""
    import json
    desc = os.path.join(ROOT, "BASELINE.json")
    ref = json.load(open(desc)).get("reference_path") if os.path.exists(desc) else None
    if not ref:
        pytest.skip("no reference location recorded")
    files = _product_modules() + [os.path.join(ROOT, "bench.py"), os.path.join(ROOT, "__graft_entry__.py")]
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    for path in files:
        assert ref not in open(path).read(), path


def test_missing_library_raises():
    from test_sequence_modeling_b200 import _lib
    with pytest.raises(RuntimeError, match="not built"):
        _lib.load(os.path.join(ROOT, "no_such_libttt.so"))
