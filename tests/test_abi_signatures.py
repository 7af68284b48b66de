"""The ctypes binding against the header, with no GPU: every prototype in
include/nosa.h has the same parameter count and the same kind of argument in
each position (pointer, 32-bit integer, 64-bit integer, size) as the argtypes
the binding installs, and the two structs have the header's fields in the
header's order and widths.  A mismatch here would pass garbage through the
ABI without any error."""

import ctypes as C
import os
import re

import pytest

from kv_cache_decode_step_b200 import build as nbuild
from kv_cache_decode_step_b200 import nosa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = open(os.path.join(ROOT, "include", "nosa.h")).read()


def _strip_comments(src):
    return re.sub(r"/\*.*?\*/", "", src, flags=re.S)


def prototypes():
    src = _strip_comments(HEADER)
    out = {}
    for m in re.finditer(r"NOSA_API\s+([\w\s\*]+?)\b(nosa_\w+)\s*\(([^)]*)\)\s*;", src):
        params = [p.strip() for p in m.group(3).split(",")]
        if params == ["void"] or params == [""]:
            params = []
        out[m.group(2)] = (m.group(1).strip(), params)
    return out


def c_kind(decl):
    """Kind of a C parameter declaration."""
    if "*" in decl or decl.split()[0] in ("nosa_stream_t",) or "nosa_stream_t" in decl:
        return "ptr"
    t = decl.replace("const ", "").split()[0]
    return {"int": "i32", "int32_t": "i32", "uint32_t": "i32", "int64_t": "i64", "size_t": "size"}[t]


def ct_kind(t):
    """Kind of a ctypes argument type."""
    if t in (C.c_void_p, C.c_char_p) or (isinstance(t, type) and issubclass(t, C._Pointer)):
        return "ptr"
    if t in (C.c_int, C.c_int32, C.c_uint32):
        return "i32"
    if t is C.c_size_t:
        return "size"
    if t in (C.c_int64, C.c_longlong):
        return "i64"
    raise AssertionError(f"unexpected ctypes type {t}")


@pytest.fixture(scope="module")
def L():
    nbuild.build()
    return nosa.lib()


def test_every_prototype_is_parsed():
    assert sorted(prototypes()) == sorted(nosa.ENTRY_POINTS)


@pytest.mark.parametrize("name", sorted(nosa.ENTRY_POINTS))
def test_argtypes_match_the_prototype(L, name):
    ret, params = prototypes()[name]
    f = getattr(L, name)
    want = [c_kind(p) for p in params]
    got = [ct_kind(t) for t in f.argtypes]
    assert got == want, (name, params, f.argtypes)
    if ret == "nosa_status":
        assert f.restype is C.c_int
    elif ret == "void":
        assert f.restype is None
    else:
        assert ret == "const char*" and f.restype is C.c_char_p


def _struct_fields(name):
    src = _strip_comments(HEADER)
    m = re.search(r"typedef struct \{([^}]*)\}\s*" + name + r"\s*;", src)
    assert m, name
    fields = []
    for decl in m.group(1).split(";"):
        decl = decl.strip()
        if decl:
            t, n = decl.rsplit(None, 1)
            fields.append((n, t))
    return fields


WIDTH = {"int": 4, "int32_t": 4, "uint32_t": 4, "int64_t": 8}


@pytest.mark.parametrize("name,cls", [("nosa_config", nosa.nosa_config), ("nosa_stats", nosa.nosa_stats)])
def test_structs_match_the_header(name, cls):
    fields = _struct_fields(name)
    assert [n for n, _ in fields] == [n for n, _ in cls._fields_]
    for (n, t), (_, ct) in zip(fields, cls._fields_):
        assert WIDTH[t] == C.sizeof(ct), (name, n, t, ct)
    assert C.sizeof(cls) == sum(WIDTH[t] for _, t in fields)  # no padding in either struct
