"""The boundary as a whole (CPU only): every compute call the C header
declares has a Python binding of the same name, and the product package
neither imports the oracle nor reaches it any other way, so no GPU call can
fall back to it."""

import ast
import os
import re

import moe_grouped_gemm_tcgen05_b200 as dg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "moe_grouped_gemm_tcgen05_b200")
HEADER = os.path.join(ROOT, "include", "dgb200.h")


def _declared():
    return re.findall(r"DG_API\s+[\w\s\*]+?\b(\w+)\s*\(", open(HEADER).read())


def test_every_compute_call_has_a_binding_of_the_same_name():
    compute = [n for n in _declared() if not n.startswith("dgb200_")]
    assert len(compute) >= 15
    missing = [n for n in compute if not callable(getattr(dg, n, None))]
    assert not missing, missing
    assert all(n in dg.__all__ for n in compute)


def test_product_package_never_reaches_the_oracle():
    for dirpath, _, files in os.walk(PKG):
        for f in files:
            if not f.endswith(".py"):
                continue
            path = os.path.join(dirpath, f)
            tree = ast.parse(open(path).read(), filename=path)
            for node in ast.walk(tree):
                if isinstance(node, ast.Import):
                    names = [a.name for a in node.names]
                elif isinstance(node, ast.ImportFrom):
                    names = [node.module or ""]
                else:
                    continue
                assert not any(n == "oracle" or n.startswith("oracle.") for n in names), (path, names)
            src = open(path).read()
            assert "import_module(\"oracle" not in src and "__import__(\"oracle" not in src, path
