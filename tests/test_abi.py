"""The C-ABI library: it loads, exports every entry point the header declares,
and its host-side argument checks answer before any device work (no GPU needed)."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "stepq.h")).read()
    return sorted(set(re.findall(r"STEPQ_API\s+[\w\s\*]+?\b(stepq_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def S():
    from quantized_delta_rule_decode_b200 import build as B
    B.build()
    import quantized_delta_rule_decode_b200 as S
    S.load_library()
    return S


def test_header_declares_the_api():
    names = _declared()
    for n in ["stepq_plan_create", "stepq_pool_alloc", "stepq_decode_step", "stepq_pack",
              "stepq_unpack", "stepq_fp32_step", "stepq_decode_readout", "stepq_decode_fitpack",
              "stepq_get_status", "stepq_last_error"]:
        assert n in names


def test_every_declared_symbol_is_exported(S):
    lib = ctypes.CDLL(S.library_path())
    for n in _declared():
        assert hasattr(lib, n), n
    # and the binding wraps each of them under the same name
    import quantized_delta_rule_decode_b200._ffi as F
    assert set(F._SIGS) == set(_declared())
    for n in _declared():
        if n != "stepq_last_error":
            assert hasattr(S, n), n


def test_plan_argument_checks(S):
    L = S.load_library()
    h = ctypes.c_void_p()
    assert L.stepq_plan_create(None, ctypes.byref(h)) == S._ffi.ERR_INVALID
    assert b"NULL" in L.stepq_last_error()
    w = np.ones((2, 128), np.float32)
    with pytest.raises(S.StepqError) as e:
        S.stepq_plan_create(128, 128, 2, 0, 0, 0, np.array([6, 5], np.uint8), w)
    assert e.value.code == S._ffi.ERR_INVALID and "bits[1]" in str(e.value)
    bad_w = w.copy()
    bad_w[1, 3] = 0.0
    with pytest.raises(S.StepqError) as e:
        S.stepq_plan_create(128, 128, 2, 0, 0, 0, np.array([6, 6], np.uint8), bad_w)
    assert e.value.code == S._ffi.ERR_INVALID
    with pytest.raises(S.StepqError) as e:
        S.stepq_plan_create(96, 96, 2, 0, 0, 0, np.array([6, 6], np.uint8), np.ones((2, 96)))
    assert e.value.code == S._ffi.ERR_UNSUPPORTED
    with pytest.raises(S.StepqError) as e:
        S.stepq_plan_create(128, 128, 2, 3, 0, 0, np.array([6, 6], np.uint8), w)
    assert e.value.code == S._ffi.ERR_INVALID


def test_other_null_checks(S):
    L = S.load_library()
    out = ctypes.c_size_t()
    assert L.stepq_workspace_bytes(None, 4, ctypes.byref(out)) == S._ffi.ERR_INVALID
    assert L.stepq_plan_slot_bytes(None, ctypes.byref(out)) == S._ffi.ERR_INVALID
    p = ctypes.c_void_p()
    assert L.stepq_pool_alloc(None, 4, None, 0, ctypes.byref(p)) == S._ffi.ERR_INVALID
    assert L.stepq_decode_step(None, None, None, 1, 1, None, None, None, None, None, None, None, 0,
                               None, None) == S._ffi.ERR_INVALID
    assert L.stepq_fp32_step(128, 128, 4, 0, 1, None, 4, None, 1, None, None, None, None, None, None,
                             None, None) == S._ffi.ERR_INVALID
    assert L.stepq_fp32_step(96, 96, 4, 0, 1, None, 4, None, 1, None, None, None, None, None, None,
                             None, None) == S._ffi.ERR_UNSUPPORTED
    assert L.stepq_get_status(None, None) == S._ffi.ERR_INVALID
    assert L.stepq_plan_destroy(None) == 0 and L.stepq_pool_free(None) == 0
