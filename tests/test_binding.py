"""The Python binding mirrors the C ABI: every function include/tplayers.h
declares has a Python function of the same name in linear_layers_b200, and
its ctypes signature has the header's parameter count.  (Host only.)"""
import os
import re

import linear_layers_b200 as tpl

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "tplayers.h")


def _declarations():
    text = open(HEADER).read()
    out = {}
    for m in re.finditer(r"^TP_API\s+[\w\s\*]+?\b(\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M | re.S):
        params = m.group(2).strip()
        n = 0 if params in ("", "void") else len([p for p in params.split(",") if p.strip()])
        out[m.group(1)] = n
    return out


def test_every_entry_point_has_a_binding_of_the_same_name():
    decl = _declarations()
    assert len(decl) >= 20
    missing = [name for name in decl if not callable(getattr(tpl, name, None))]
    assert not missing, missing


def test_ctypes_signatures_match_the_header():
    decl = _declarations()
    for name, n in decl.items():
        assert name in tpl._SIGS, name
        assert len(tpl._SIGS[name][0]) == n, (name, len(tpl._SIGS[name][0]), n)
