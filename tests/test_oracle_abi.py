"""The oracle's own C entry points (test infrastructure): the ctypes argument lists in
oracle/__init__.py have as many entries as the C definitions have parameters, so a
parameter added on one side only fails here rather than reading garbage."""
import os
import re

import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "lightning_oracle.cpp")


def test_oracle_argument_counts_match_definitions():
    src = open(SRC).read()
    body = src[src.index('extern "C" {'):]
    body = re.sub(r"//[^\n]*", "", body)
    defs = dict(re.findall(r"\bint\s+(oracle_\w+)\s*\(([^)]*)\)\s*\{", body))
    assert "oracle_backward_znorm_packed" in defs and "oracle_transform_backward" in defs
    lib = oracle._get()
    for name, params in defs.items():
        params = params.strip()
        n = 0 if params in ("", "void") else len(params.split(","))
        argtypes = getattr(lib, name).argtypes
        assert argtypes is not None and len(argtypes) == n, (name, n, argtypes)
