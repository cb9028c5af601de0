"""CPU checks of the C ABI library: it loads without a GPU, exports every symbol that
include/svdq.h declares, and its pure host helpers follow the documented storage sizes."""
import os
import re

import pytest

from tests.conftest import ROOT


def _declared():
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    return sorted(set(re.findall(r"SVDQ_API[^;]*?\b(svdq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    from bit_rank_compensated_b200 import build, svdq

    if not os.path.exists(svdq.LIB_PATH):
        build.build()
    return svdq.load()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("svdq_prepare_weights", "svdq_quant_act_lora_down", "svdq_gemm_w4a4_lora_up"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    from bit_rank_compensated_b200 import svdq

    for name in _declared():
        assert hasattr(lib, name), name
    assert sorted(svdq.EXPORTED) == _declared()


def test_host_size_helpers(lib):
    assert lib.svdq_weight_scale_bytes(9216, 3072) == 9216 * 192
    assert lib.svdq_weight_scale_bytes(272, 64) == 512 * 4
    assert lib.svdq_act_scale_bytes(4608, 3072) == 4608 * 192
    assert lib.svdq_act_scale_bytes(1, 64) == 128 * 4
    assert lib.svdq_act_scale_bytes(0, 64) == 0
    assert lib.svdq_version() >= 100


def test_status_strings(lib):
    assert lib.svdq_status_string(0) == b"ok"
    assert b"10.0" in lib.svdq_status_string(2)
    assert lib.svdq_status_string(99) == b"unknown status"


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    from bit_rank_compensated_b200 import svdq

    monkeypatch.setattr(svdq, "_lib", None)
    monkeypatch.setattr(svdq, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        svdq.load()


def _declared_params():
    """{name: [parameter declarations]} parsed from include/svdq.h."""
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"SVDQ_API\s+[^;(]*?\b(svdq_\w+)\s*\(([^)]*)\)\s*;", src, flags=re.S):
        params = [p.strip() for p in m.group(2).split(",") if p.strip()]
        out[m.group(1)] = [] if params == ["void"] else params
    return out


def test_binding_argument_counts_match_the_header(lib):
    # every declared entry point is bound with as many ctypes arguments as the header has
    # parameters, and pointer parameters are bound as pointers
    import ctypes

    decl = _declared_params()
    assert sorted(decl) == _declared()
    for name, params in decl.items():
        f = getattr(lib, name)
        assert f.argtypes is not None, name
        assert len(f.argtypes) == len(params), (name, params, f.argtypes)
        for p, t in zip(params, f.argtypes):
            if "*" in p:
                assert t is ctypes.c_void_p or issubclass(t, (ctypes._Pointer, ctypes.c_char_p)), (name, p, t)
            elif re.match(r"(const\s+)?(int|uint32_t)\b", p):
                assert t in (ctypes.c_int, ctypes.c_uint32), (name, p, t)
            elif re.match(r"(const\s+)?float\b", p):
                assert t is ctypes.c_float, (name, p, t)


def _declared_returns():
    """{name: return type} parsed from include/svdq.h."""
    src = open(os.path.join(ROOT, "include", "svdq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return {m.group(2): " ".join(m.group(1).split())
            for m in re.finditer(r"SVDQ_API\s+([^;(]*?)\b(svdq_\w+)\s*\(", src, flags=re.S)}


def test_binding_types_match_the_header(lib):
    # every parameter and return type is bound with a ctypes type of the same width: size_t as
    # c_size_t (a 32-bit binding would truncate workspace sizes), enums and int as c_int
    import ctypes

    scalar = {"int": (ctypes.c_int,), "uint32_t": (ctypes.c_uint32, ctypes.c_int), "float": (ctypes.c_float,),
              "size_t": (ctypes.c_size_t,), "svdq_status": (ctypes.c_int,)}
    for name, params in _declared_params().items():
        f = getattr(lib, name)
        for p, t in zip(params, f.argtypes):
            if "*" in p:
                continue  # pointers: checked by the count test
            base = re.sub(r"^const\s+", "", p).split()[0]
            assert base in scalar, (name, p)
            assert t in scalar[base], (name, p, t)
    for name, ret in _declared_returns().items():
        f = getattr(lib, name)
        if ret.endswith("*"):
            assert f.restype is ctypes.c_char_p, (name, ret, f.restype)
        else:
            base = re.sub(r"^const\s+", "", ret).split()[-1]
            assert base in scalar, (name, ret)
            assert f.restype in scalar[base], (name, ret, f.restype)
