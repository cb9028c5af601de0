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
