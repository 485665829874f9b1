"""The binding's ctypes signatures agree with include/fftconv.h: for every
exported call, the same number of arguments, pointer arguments as pointers,
64-bit integers as 64-bit, and the matching return type."""
import ctypes
import os
import re

from fft_long_convolution_causal_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fftconv.h")


def _declarations():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"FFTCONV_API\s+([\w\s\*]+?)\b(\w+)\s*\(([^)]*)\)\s*;", text):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        args = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        out[name] = (ret, args)
    return out


def _ret_ctype(ret):
    ret = " ".join(ret.split())
    return {"size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p, "double": ctypes.c_double,
            "fftconv_status": ctypes.c_int, "int": ctypes.c_int, "void": None}[ret.replace(" *", "*")]


def _arg_ok(decl, ctype):
    d = " ".join(decl.split())
    if "*" in d or d.startswith("fftconv_plan_t ") or d.startswith("void*"):
        # pointers, handles and streams: a pointer-sized type
        return ctypes.sizeof(ctype) == ctypes.sizeof(ctypes.c_void_p) and ctype not in (ctypes.c_int64,
                                                                                         ctypes.c_uint64)
    if d.startswith("int64_t"):
        return ctype is ctypes.c_int64
    if d.startswith("uint32_t"):
        return ctype is ctypes.c_uint32
    if d.startswith(("int ", "fftconv_dtype", "fftconv_status")):
        return ctype is ctypes.c_int
    raise AssertionError(f"unexpected parameter type in the header: {decl}")


def test_every_declaration_has_a_matching_signature():
    decls = _declarations()
    assert len(decls) >= 30
    for name, (ret, args) in decls.items():
        assert name in binding._SIGS, name
        restype, argtypes = binding._SIGS[name]
        assert restype == _ret_ctype(ret), (name, ret, restype)
        assert len(argtypes) == len(args), (name, args, argtypes)
        for decl, ct in zip(args, argtypes):
            assert _arg_ok(decl, ct), (name, decl, ct)


def test_no_signature_without_a_declaration():
    decls = _declarations()
    assert set(binding._SIGS) <= set(decls), sorted(set(binding._SIGS) - set(decls))
