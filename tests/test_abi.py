"""The C-ABI library loads, exports every symbol include/owq.h declares, and rejects bad
arguments on the host (no GPU needed for any of these)."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT


def _gpu_present():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="module")
def owq():
    from weight_only_mixed_owq_b200 import build
    build.build()
    import weight_only_mixed_owq_b200 as m
    return m


def _declared_functions():
    txt = open(os.path.join(ROOT, "include", "owq.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(owq_[a-z_]+)\s*\(", txt)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for must in ("owq_pack", "owq_gemv", "owq_gemm", "owq_quantize", "owq_dequant"):
        assert must in names


def test_library_exports_every_declared_symbol(owq):
    lib = ctypes.CDLL(owq.LIB_PATH)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert {p[0] for p in owq.PROTOTYPES} == set(_declared_functions())


def test_debug_bounds_variant_exports_every_declared_symbol(owq):
    """The debug-bounds build (built by __graft_entry__.build()) exports the same boundary and
    names itself in owq_version; OWQ_INJECT_BOUNDS is refused by the default build."""
    from weight_only_mixed_owq_b200 import build
    path = build.LIB_BOUNDS
    if not os.path.exists(path):
        pytest.skip("debug-bounds variant not built (python -m weight_only_mixed_owq_b200.build --debug-bounds)")
    if not build.up_to_date(path):   # built from older sources: rebuild it first
        build.build(debug_bounds=True)
    lib = ctypes.CDLL(path)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    lib.owq_version.restype = ctypes.c_char_p
    assert lib.owq_version().decode().endswith("+debug-bounds")
    assert owq.owq_debug_inject(owq.OWQ_INJECT_BOUNDS, 1) == 12   # OWQ_ERR_ARG in the default build


def test_status_strings_and_version(owq):
    for code, name in owq.STATUS_NAMES.items():
        assert owq.owq_status_string(code).startswith(name)
    assert re.match(r"^\d+\.\d+\.\d+$", owq.owq_version())


def test_host_validation_rejects_bad_arguments(owq):
    A = 0x10000  # never dereferenced: every call below fails validation first
    # NULL pointers
    assert owq.owq_quantize(None, A, 16, 128, 8, 3, 128, 1, A, A, A, A, A) == 1
    st, h = owq.owq_pack(None, 16, 128, 3, 128, A, A, A, 1, A)
    assert st == 1 and h is None
    # bits, group, shape
    assert owq.owq_quantize(A, A, 16, 128, 8, 5, 128, 1, A, A, A, A, A) == 3
    assert owq.owq_quantize(A, A, 16, 256, 8, 3, 64, 1, A, A, A, A, A) == 4
    assert owq.owq_quantize(A, A, 16, 100, 8, 3, 100, 1, A, A, A, A, A) == 2
    assert owq.owq_quantize(A, A, 0, 128, 8, 3, 128, 1, A, A, A, A, A) == 2
    assert owq.owq_quantize(A, A, 16, 128, 0, 3, 128, 1, A, A, A, A, A) == 2
    assert owq.owq_quantize(A, A, 16, 128, 8, 3, 128, 129, A, A, A, A, A) == 2
    # alignment
    assert owq.owq_quantize(A + 2, A, 16, 128, 8, 3, 128, 1, A, A, A, A, A) == 6
    # handles
    assert owq.owq_gemv(None, A, A, 1) == 10
    assert owq.owq_gemv(A, A, A, 1) == 10
    assert owq.owq_gemm(A, A, A, 64) == 10
    assert owq.owq_dequant(A, A) == 10
    assert owq.owq_weak_grad(A, A, A, A, 1) == 10
    assert owq.owq_weak_grad(None, A, A, A, 16) == 10
    assert owq.owq_input_grad(A, A, A, 1) == 10
    assert owq.owq_input_grad(None, A, A, 16) == 10
    assert owq.owq_layer_free(A) == 10
    assert owq.owq_layer_free(None) == 0
    assert owq.owq_layer_info(A)[0] == 10
    assert owq.owq_layer_bytes(A)[0] == 10
    # fault-injection hook: unknown kinds and empty wait bounds are refused
    assert owq.owq_debug_inject(3, 1000) == 12
    assert owq.owq_debug_inject(-1, 1000) == 12
    assert owq.owq_debug_inject(owq.OWQ_INJECT_GEMV_TAG, 0) == 12
    assert owq.owq_debug_inject(owq.OWQ_INJECT_NONE, 0) == 0
    # parameter search
    assert owq.owq_search_params(None, 16, 128, 3, 128, A, 1, A, A) == 1
    assert owq.owq_search_params(A, 16, 128, 5, 128, A, 1, A, A) == 3
    assert owq.owq_search_params(A, 16, 256, 3, 64, A, 1, A, A) == 4
    assert owq.owq_search_params(A + 8, 16, 128, 3, 128, A, 1, A, A) == 6
    # OPTQ
    assert owq.owq_optq(None, A, 16, 128, 8, 3, 128, A, 1, A, A, 0.01, A, A) == 1
    assert owq.owq_optq(A, A, 16, 128, 0, 3, 128, A, 1, A, A, 0.01, A, A) == 2
    assert owq.owq_optq(A, A, 16, 128, 8, 3, 128, A, 1, A, A, -1.0, A, A) == 12
    assert owq.owq_optq(A, A, 16, 128, 8, 3, 128, A, 1, A, A, float("nan"), A, A) == 12
    assert owq.owq_optq(A, A + 2, 16, 128, 8, 3, 128, A, 1, A, A, 0.01, A, A) == 6
    assert owq.owq_quantize_optq(A, A, 16, 128, 8, 3, 128, 1, -0.5, A, A, A, A, A) == 12
    assert owq.owq_quantize_optq(None, A, 16, 128, 8, 3, 128, 1, 0.01, A, A, A, A, A) == 1
    # storage-favoured stream: host word count, NULL pointers, shapes, alignment
    assert owq.owq_storage_words(4096, 3, 32) == (0, ((4096 - 32) * 3 + 31) // 32)
    assert owq.owq_storage_words(11008, 4, 86) == (0, ((11008 - 86) * 4 + 31) // 32)
    assert owq.owq_storage_words(4096, 5, 32)[0] == 3
    assert owq.owq_storage_words(4096, 3, 1025)[0] == 2
    assert owq.owq_storage_pack(None, 16, 128, 3, A, 1, A) == 1
    assert owq.owq_storage_pack(A, 16, 100, 3, A, 1, A) == 2
    assert owq.owq_storage_pack(A + 4, 16, 128, 3, A, 1, A) == 6
    assert owq.owq_storage_unpack(A, 16, 256, 3, 64, A, 1, A, A) == 4
    assert owq.owq_storage_unpack(A, 16, 128, 3, 128, None, 1, A, A) == 1
    st, h = owq.owq_pack_storage(A, 16, 128, 4, 128, A, A, None, 1, A)
    assert st == 1 and h is None


@pytest.mark.skipif(_gpu_present(), reason="checks the no-device path; needs a machine without a GPU")
def test_valid_arguments_without_device_report_device_error(owq):
    A = 0x10000
    assert owq.owq_quantize(A, A, 16, 128, 8, 3, 128, 1, A, A, A, A, A) == 11
    st, _ = owq.owq_pack(A, 16, 128, 3, 128, A, A, A, 1, A)
    assert st == 11
