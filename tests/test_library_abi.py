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
