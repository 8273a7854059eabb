"""The binding's ctypes signatures agree with the C declarations in include/w4a16.h, parameter by
parameter (a mismatch, e.g. int where the header has int64_t, would pass wrong values silently)."""
import ctypes
import os
import re

from weight_only_int4_06_b200 import w4a16 as B

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "w4a16.h")

SCALARS = {"int64_t": ctypes.c_int64, "uint64_t": ctypes.c_uint64, "int": ctypes.c_int, "size_t": ctypes.c_size_t, "double": ctypes.c_double,
           "w4_status": ctypes.c_int}


def _declarations():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    text = re.sub(r"#.*", "", text)
    out = {}
    for m in re.finditer(r"(?:const\s+)?(\w+\s*\**)\s*(\w+)\s*\(([^)]*)\)\s*;", text):
        ret, name, params = m.group(1), m.group(2), m.group(3)
        if name in ("if", "while"):
            continue
        ps = [p.strip() for p in params.split(",") if p.strip() and p.strip() != "void"]
        out[name] = (ret.strip(), ps)
    return out


def _expected(param):
    p = re.sub(r"\bconst\b", "", param).strip()
    stars = p.count("*")
    base = p.replace("*", " ").split()[0]
    if stars == 0:
        return SCALARS[base]
    if base == "size_t":
        return ctypes.POINTER(ctypes.c_size_t)
    if base == "int":  # host int outputs of the queries
        return ctypes.POINTER(ctypes.c_int)
    return ctypes.c_void_p


def test_every_declared_function_has_a_matching_signature():
    decls = _declarations()
    assert len(decls) >= 25
    for name, (ret, params) in decls.items():
        assert name in B.SIGNATURES, name
        res, args = B.SIGNATURES[name]
        assert len(args) == len(params), (name, len(args), len(params))
        for i, (a, p) in enumerate(zip(args, params)):
            want = _expected(p)
            same = a is want or (isinstance(a, type) and isinstance(want, type) and a.__name__ == want.__name__)
            assert same, (name, i, p, a, want)
        if ret.startswith("w4_status"):
            assert res is ctypes.c_int, name
