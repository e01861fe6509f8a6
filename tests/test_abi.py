"""The C-ABI library loads and exports every function the headers declare;
argument validation happens on the host (no GPU needed for these calls)."""
import ctypes
import glob
import os
import re

import pytest
import torch

import streaming_top_b200 as si

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names += re.findall(r"SI_API\s+[\w\s\*]+?\b(si_\w+)\s*\(", src)
    return sorted(set(names))


def test_headers_declare_the_entry_points():
    names = declared_functions()
    for n in ("si_indexer_topk", "si_indexer_topk_ex", "si_indexer_materialize",
              "si_indexer_workspace_size", "si_device_status", "si_status_string", "si_last_error",
              "si_version"):
        assert n in names


@pytest.mark.parametrize("name", declared_functions())
def test_library_exports(name):
    assert hasattr(si.lib(), name), name


def declared_prototypes():
    """{name: (return type, [parameter types])} of every SI_API function."""
    out = {}
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for ret, name, params in re.findall(r"SI_API\s+([\w\s\*]+?)\s*\b(si_\w+)\s*\(([^)]*)\)", src):
            ps = [" ".join(p.split()) for p in params.split(",")]
            ps = [] if ps == ["void"] else ps
            # drop the parameter name: the last identifier, unless the type is all there is
            types = [re.sub(r"\s*\b\w+$", "", p) if re.search(r"[\w\*]\s+\w+$", p) else p for p in ps]
            out[name] = (" ".join(ret.split()), types)
    return out


def _ctype_ok(c_type: str, ct) -> bool:
    c_type = c_type.replace("const ", "")
    if c_type == "float":
        return ct is ctypes.c_float
    if "*" in c_type:
        if c_type == "char*" or c_type == "char *":
            return ct is ctypes.c_char_p
        return ct is ctypes.c_void_p or (isinstance(ct, type) and issubclass(ct, ctypes._Pointer))
    return {"int": ctypes.c_int, "si_status": ctypes.c_int, "int64_t": ctypes.c_int64,
            "size_t": ctypes.c_size_t, "unsigned long long": ctypes.c_ulonglong}[c_type] is ct


@pytest.mark.parametrize("name", sorted(declared_prototypes()))
def test_binding_prototypes_match_the_headers(name):
    """The ctypes prototypes of the binding have the headers' arity and types,
    so a change of either side is caught here rather than by a wrong call."""
    ret, params = declared_prototypes()[name]
    f = getattr(si.lib(), name)
    assert f.argtypes is not None, f"{name}: the binding sets no argtypes"
    assert len(f.argtypes) == len(params), (name, params, f.argtypes)
    for c_type, ct in zip(params, f.argtypes):
        assert _ctype_ok(c_type, ct), (name, c_type, ct)
    if ret == "void":
        assert f.restype is None, name
    else:
        assert _ctype_ok(ret, f.restype), (name, ret, f.restype)


def test_options_struct_matches_the_header():
    src = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "streaming_top.h")).read(), flags=re.S)
    body = re.search(r"typedef struct si_options \{(.*?)\} si_options;", src, flags=re.S).group(1)
    fields = [re.search(r"(\w+)\s*;", d).group(1) for d in body.split(";") if d.strip() for d in [d + ";"]]
    assert fields == [f for f, _ in si.Options._fields_]


def test_status_strings_and_version():
    L = si.lib()
    assert L.si_status_string(si.SI_ERR_TIMEOUT) == b"SI_ERR_TIMEOUT"
    assert L.si_status_string(0) == b"SI_OK"
    assert si.version() >= 100


# Fake, 16-byte aligned addresses: every call below is rejected by host-side
# validation before any CUDA call, so nothing ever dereferences them.
P = 4096


def _call(q=P, kc=P, w=P, B=1, S=64, T=16, H=64, D=128, m=4, k=8, out=P, opt=None):
    o = ctypes.byref(opt) if opt is not None else None
    return si.lib().si_indexer_topk_ex(q, kc, w, B, S, T, H, D, m, k, out, None, None, o)


@pytest.mark.parametrize("kw,status", [
    ({"q": None}, si.SI_ERR_INVALID_ARGUMENT),
    ({"out": None}, si.SI_ERR_INVALID_ARGUMENT),
    ({"S": 0}, si.SI_ERR_INVALID_ARGUMENT),
    ({"k": 0}, si.SI_ERR_INVALID_ARGUMENT),
    ({"m": 0}, si.SI_ERR_INVALID_ARGUMENT),
    ({"q": P + 8}, si.SI_ERR_INVALID_ARGUMENT),
    ({"D": 64}, si.SI_ERR_UNSUPPORTED),
    ({"H": 32}, si.SI_ERR_UNSUPPORTED),
    ({"k": 4096}, si.SI_ERR_UNSUPPORTED),
])
def test_validation(kw, status):
    assert _call(**kw) == status
    assert si.lib().si_last_error()  # a message was recorded


@pytest.mark.parametrize("field,value", [("key_tile", 100), ("key_tile", 2048), ("query_chunk", 6),
                                         ("query_chunk", -4), ("dtype", 7)])
def test_option_validation(field, value):
    o = si.Options()
    setattr(o, field, value)
    assert _call(opt=o) == si.SI_ERR_INVALID_ARGUMENT


def test_fp8_needs_scales():
    o = si.Options()
    o.dtype = si.SI_DTYPE_FP8_E4M3
    assert _call(opt=o) == si.SI_ERR_INVALID_ARGUMENT


def test_workspace_size():
    # enough 4-query units for any GPU: no split-key partials, no scratch
    assert si.workspace_size(1, 8192, 2048, 64, 128, 4, 64, materialize=False) == 0
    # few units: room for the split-key partials (a bound independent of row0)
    small = si.workspace_size(1, 64, 1 << 16, 64, 128, 4, 64, materialize=False)
    assert small >= 4 * 148 * 64 * 8
    assert si.workspace_size(1, 64, 1 << 16, 64, 128, 4, 64, mxfp4=True) == small + (1 << 16) * 128 * 2 + 256
    need = si.workspace_size(1, 1024, 256, 64, 128, 4, 64, materialize=True)
    assert need >= 4 * 1024 * 256 * 65


@pytest.mark.parametrize("idx,score,rows,k,status", [
    (P, P, 4, 0, si.SI_ERR_INVALID_ARGUMENT),
    (P, P, 4, 4096, si.SI_ERR_INVALID_ARGUMENT),
    (P, P, -1, 8, si.SI_ERR_INVALID_ARGUMENT),
    (None, P, 4, 8, si.SI_ERR_INVALID_ARGUMENT),
    (P, None, 4, 8, si.SI_ERR_INVALID_ARGUMENT),
    (P + 2, P, 4, 8, si.SI_ERR_INVALID_ARGUMENT),
    (None, None, 0, 8, si.SI_OK),  # nothing to sort: no device work at all
])
def test_row_sort_validation(idx, score, rows, k, status):
    assert si.lib().si_sort_topk_rows(idx, score, rows, k, None) == status


def test_row_range_validation():
    L = si.lib()
    o = si.Options()
    # a negative first row is refused on the host, before any device work
    assert L.si_indexer_topk_rows(P, P, P, 1, -4, 64, 16, 64, 128, 4, 8, P, None, None,
                                  ctypes.byref(o)) == si.SI_ERR_INVALID_ARGUMENT
    assert L.si_indexer_topk_rows(P, P, P, 1, 0x7FFFFFF0, 64, 16, 64, 128, 4, 8, P, None, None,
                                  ctypes.byref(o)) == si.SI_ERR_UNSUPPORTED


def test_mxfp4_validation():
    L = si.lib()
    o = si.Options()
    o.dtype = si.SI_DTYPE_MXFP4_KEYS
    args = (P, P, P, 1, 64, 16, 64, 128, 4, 8, P, None, None, ctypes.byref(o))
    assert L.si_indexer_topk_ex(*args) == si.SI_ERR_INVALID_ARGUMENT  # no block scales
    o.kc_mx_scale = P
    o.workspace, o.workspace_bytes = P, 64  # too small for the decoded keys
    assert L.si_indexer_topk_ex(*args) == si.SI_ERR_INVALID_ARGUMENT
    o.workspace, o.workspace_bytes = None, 0
    o.dtype = si.SI_DTYPE_BF16
    base = L.si_indexer_workspace_size(2, 64, 16, 64, 128, 4, 8, 0, ctypes.byref(o))
    o.dtype = si.SI_DTYPE_MXFP4_KEYS
    assert L.si_indexer_workspace_size(2, 64, 16, 64, 128, 4, 8, 0, ctypes.byref(o)) == base + 2 * 16 * 128 * 2 + 256
    assert L.si_mxfp4_to_bf16(P, P, 4, 48, P, None) == si.SI_ERR_INVALID_ARGUMENT  # D % 32
    assert L.si_mxfp4_to_bf16(P, P, -1, 128, P, None) == si.SI_ERR_INVALID_ARGUMENT
    assert L.si_mxfp4_to_bf16(P + 8, P, 4, 128, P, None) == si.SI_ERR_INVALID_ARGUMENT  # alignment
    assert L.si_mxfp4_to_bf16(P, P, 0, 128, P, None) == si.SI_OK  # nothing to do


def test_mxfp4_options_keep_their_dtype():
    """The binding's option marshalling for MXFP4 keys (CPU tensors stand in
    for device ones: only shapes, dtypes and pointers are read)."""
    q = torch.zeros((1, 8, 64, 128), dtype=torch.bfloat16)
    kc = torch.zeros((1, 2, 64), dtype=torch.uint8)
    ms = torch.zeros((1, 2, 4), dtype=torch.uint8)
    o = si._options(q, kc, None, None, 0, 0, kc_mx_scale=_Cuda(ms))
    assert o.dtype == si.SI_DTYPE_MXFP4_KEYS and o.kc_mx_scale == ms.data_ptr()
    o = si._options(q, torch.zeros((1, 2, 128), dtype=torch.bfloat16), None, None, 0, 0)
    assert o.dtype == si.SI_DTYPE_BF16 and not o.kc_mx_scale
    with pytest.raises(ValueError):
        si._options(q, torch.zeros((1, 2, 128), dtype=torch.uint8), None, None, 0, 0, kc_mx_scale=_Cuda(ms))


class _Cuda:
    """A CPU tensor that reports itself as a CUDA one (shape checks only)."""

    def __init__(self, t):
        self._t = t
        self.is_cuda = True
        self.dtype, self.shape = t.dtype, t.shape

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return self._t.data_ptr()


def test_two_stage_validation():
    L = si.lib()
    args = [P, P, P, 1, 64, 64, 64, 128, 4, 8]
    assert L.si_indexer_topk_two_stage(*args, 0, 16, P, P, None, None) == si.SI_ERR_INVALID_ARGUMENT  # block 0
    assert L.si_indexer_topk_two_stage(*args, 8, 4096, P, P, None, None) == si.SI_ERR_INVALID_ARGUMENT
    assert L.si_indexer_topk_two_stage(*args, 8, 16, P, None, None, None) == si.SI_ERR_INVALID_ARGUMENT
    o = si.Options()
    o.dtype = si.SI_DTYPE_FP8_E4M3
    assert L.si_indexer_topk_two_stage(*args, 8, 16, P, P, None, ctypes.byref(o)) == si.SI_ERR_UNSUPPORTED
    assert L.si_indexer_topk_two_stage(P, P, P, 1, 64, 64, 32, 128, 4, 8, 8, 16, P, P, None, None) == \
        si.SI_ERR_UNSUPPORTED  # H_I = 32
    assert si.two_stage_workspace_size(1, 64, 64, 8, 16, 0) > 0
    assert si.two_stage_workspace_size(1, 64, 64, 0, 16, 0) == 0
