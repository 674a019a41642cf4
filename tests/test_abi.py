"""The C-ABI library loads on a machine without a GPU and exports every entry point that
include/rptq.h declares; host-side argument validation needs no GPU either."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(rptq_[a-z_0-9]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def rlib():
    from post_activation_quantization_b200 import build, rptq
    build.build()
    return rptq.lib()


def test_every_declared_symbol_is_exported(rlib):
    from post_activation_quantization_b200 import rptq
    names = _declared_functions()
    assert "rptq_ln_reorder_quant" in names and len(names) >= 9
    for n in names:
        assert hasattr(rlib, n), n
    assert set(names) == set(rptq.SIGNATURES)


def test_status_strings_and_version(rlib):
    assert rlib.rptq_version() == 100
    assert rlib.rptq_status_string(0) == b"ok"
    for st in (-1, -2, -3, -4, -5):
        assert rlib.rptq_status_string(st) != b"unknown status"


def test_workspace_size_rules(rlib):
    assert rlib.rptq_kmeans_workspace_size(12288, 64) > 0
    assert rlib.rptq_kmeans_workspace_size(8, 9) == 0      # g > C
    assert rlib.rptq_kmeans_workspace_size(0, 1) == 0
    assert rlib.rptq_kmeans_workspace_size(20000, 8) == 0  # C over the maximum


def test_host_validation_rejects_before_any_launch(rlib):
    """Invalid calls are refused on the host (no CUDA context is touched)."""
    P = ctypes.c_void_p
    fake = P(16 * 1024)  # never dereferenced: validation fails first
    # bits not in {3, 4}
    assert rlib.rptq_ln_reorder_quant(fake, 2, 4, 64, fake, fake, 1e-5, fake, fake, fake, fake, 8, 5,
                                      fake, None, None) == -2
    # C not a multiple of 8
    assert rlib.rptq_ln_reorder_quant(fake, 2, 4, 60, fake, fake, 1e-5, fake, fake, fake, fake, 8, 3,
                                      fake, None, None) == -2
    # neither codes nor ln_out
    assert rlib.rptq_ln_reorder_quant(fake, 2, 4, 64, fake, fake, 1e-5, fake, fake, fake, fake, 8, 3,
                                      None, None, None) == -1
    # misaligned x
    assert rlib.rptq_ln_reorder_quant(P(16 * 1024 + 2), 2, 4, 64, fake, fake, 1e-5, fake, fake, fake,
                                      fake, 8, 3, fake, None, None) == -1
    # unsupported dtype
    assert rlib.rptq_calib_minmax(fake, 7, 4, 64, None, None, 1e-5, fake, fake, 0, None) == -2
    # gamma without beta
    assert rlib.rptq_calib_minmax(fake, 2, 4, 64, fake, None, 1e-5, fake, fake, 0, None) == -1
    # kmeans: g > C, bad bits, missing workspace
    assert rlib.rptq_kmeans(fake, fake, 8, 9, 1, 3, fake, fake, fake, fake, fake, fake, fake, fake,
                            1 << 20, None) == -1
    assert rlib.rptq_kmeans(fake, fake, 64, 8, 1, 2, fake, fake, fake, fake, fake, fake, fake, fake,
                            1 << 20, None) == -2
    assert rlib.rptq_kmeans(fake, fake, 64, 8, 1, 3, fake, fake, fake, fake, fake, fake, fake, None,
                            1 << 20, None) == -3
    assert rlib.rptq_kmeans(fake, fake, 64, 8, 1, 3, fake, fake, fake, fake, fake, fake, fake, fake,
                            16, None) == -3
    # kv: D not a multiple of 8, neither k nor v
    assert rlib.rptq_kv_quant(fake, fake, 1, 1, 2, 4, 12, fake, fake, fake, fake, fake, fake, 4, 3,
                              fake, fake, None) == -2
    assert rlib.rptq_kv_quant(None, None, 1, 1, 2, 4, 16, fake, fake, fake, fake, fake, fake, 4, 3,
                              fake, fake, None) == -1
    # dequant: bad layout
    assert rlib.rptq_dequant(fake, 5, 4, 64, 0, 0, fake, fake, fake, 8, 3, fake, 0, None) == -1
    # LayerNorm plan: bad bits, no plan buffer; planned launch: C not a multiple of 32
    assert rlib.rptq_ln_quant_plan(fake, fake, fake, fake, fake, fake, 64, 8, 5, fake, None) == -2
    assert rlib.rptq_ln_quant_plan(fake, fake, fake, fake, fake, fake, 64, 8, 3, None, None) == -1
    assert rlib.rptq_ln_reorder_quant_planned(fake, 2, 4, 40, 1e-5, fake, 3, fake, None) == -2
    # linear layer: C not a multiple of 64, no rows of weights, bad bits, too many outputs
    assert rlib.rptq_linear_prepare(fake, fake, 8, 96, fake, fake, fake, fake, 4, fake, fake, fake, None) == -2
    assert rlib.rptq_linear_prepare(fake, fake, 0, 128, fake, fake, fake, fake, 4, fake, fake, fake, None) == -1
    assert rlib.rptq_reordered_linear(fake, 4, 128, 5, fake, fake, fake, fake, 8, fake, None) == -2
    assert rlib.rptq_reordered_linear(fake, 4, 128, 3, fake, fake, fake, fake, 65535 * 256 + 1, fake, None) == -1
    assert rlib.rptq_device_error(None, None) == -1


def test_empty_problems_succeed_on_the_host(rlib):
    """Empty problems are valid no-ops: they return before any CUDA call (this runs without a
    GPU) and accept NULL data pointers, as an empty tensor provides."""
    P = ctypes.c_void_p
    fake = P(16 * 1024)  # tables: never dereferenced
    # T = 0 rows, x / codes / ln_out NULL
    assert rlib.rptq_ln_reorder_quant(None, 2, 0, 64, fake, fake, 1e-5, fake, fake, fake, fake, 8, 3,
                                      None, None, None) == 0
    # S = 0 and B = 0 caches
    assert rlib.rptq_kv_quant(None, None, 1, 2, 3, 0, 64, None, None, None, None, None, None, 4, 3,
                              None, None, None) == 0
    assert rlib.rptq_kv_quant(None, None, 1, 0, 3, 5, 64, None, None, None, None, None, None, 4, 3,
                              None, None, None) == 0
    # n0 = 0 rows; S = 0 positions of a BHSD cache
    assert rlib.rptq_dequant(None, 0, 0, 64, 0, 0, fake, fake, fake, 8, 3, None, 0, None) == 0
    assert rlib.rptq_dequant(None, 1, 2, 3, 0, 64, fake, fake, fake, 8, 3, None, 0, None) == 0
    # T = 0 tokens through the planned launch and the linear layer
    assert rlib.rptq_ln_reorder_quant_planned(None, 2, 0, 64, 1e-5, fake, 3, None, None) == 0
    assert rlib.rptq_reordered_linear(None, 0, 128, 3, fake, fake, fake, fake, 8, None, None) == 0
    # ... but an empty problem with an invalid shape is still refused
    assert rlib.rptq_ln_reorder_quant(None, 2, 0, 60, fake, fake, 1e-5, fake, fake, fake, fake, 8, 3,
                                      None, None, None) == -2


def _prototypes():
    """name -> list of C parameter types, parsed from the prototypes in include/*.h."""
    src = "".join(open(os.path.join(ROOT, "include", h)).read()
                  for h in sorted(os.listdir(os.path.join(ROOT, "include"))) if h.endswith(".h"))
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    out = {}
    for m in re.finditer(r"(?:\bint\s+|\bsize_t\s+|\bconst char\s*\*\s*)(rptq_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(1)] = params
    return out


def _ctype_of(param: str):
    t = re.sub(r"\s+", " ", param.rsplit(" ", 1)[0] if "*" not in param else param[: param.rindex("*") + 1])
    if "*" in t or t.endswith("rptq_stream_t"):
        return ctypes.c_void_p if "char" not in t else ctypes.c_char_p
    return {"int": ctypes.c_int, "int64_t": ctypes.c_int64, "size_t": ctypes.c_size_t,
            "float": ctypes.c_float, "unsigned long long": ctypes.c_ulonglong}[t.replace("const ", "").strip()]


def test_binding_argument_types_match_the_header():
    """The Python binding's ctypes signature of every entry point has the header's parameter
    count and, position by position, a ctypes type of the same size and kind."""
    from post_activation_quantization_b200 import rptq
    protos = _prototypes()
    assert set(protos) == set(rptq.SIGNATURES)
    for name, params in protos.items():
        _, argtypes = rptq.SIGNATURES[name]
        assert len(argtypes) == len(params), name
        for i, (p, a) in enumerate(zip(params, argtypes)):
            want = _ctype_of(p)
            if want is ctypes.c_void_p:  # any pointer: void*, typed pointers, the stream handle
                assert a is ctypes.c_void_p or hasattr(a, "_type_") and ctypes.sizeof(a) == ctypes.sizeof(ctypes.c_void_p), (name, i, p)
            else:
                assert a is want or ctypes.sizeof(a) == ctypes.sizeof(want) and a._type_ == want._type_, (name, i, p, a)
