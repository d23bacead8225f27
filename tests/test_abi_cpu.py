"""C-ABI checks that need no GPU: the library loads, exports every function that
include/qg.h declares, and rejects bad arguments before touching a device."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

import int4_quantized_gemm_b200 as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qg.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qg_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_hot_path_entry_points():
    names = _declared_functions()
    for n in ("qg_quantize_rowwise_int8", "qg_gemm_w8a8", "qg_gemm_w8a16", "qg_gemm_w4a16",
              "qg_quantize_block_asym4"):
        assert n in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", qg.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s(qg_\w+)", out))
    declared = set(_declared_functions())
    assert declared <= exported, declared - exported
    assert set(qg.SIGNATURES) == declared


def test_debug_library_exports_the_same_symbols():
    if not os.path.exists(qg.DEBUG_LIB_PATH):
        pytest.skip("libqg_debug.so not built")
    out = subprocess.run(["nm", "-D", "--defined-only", qg.DEBUG_LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    assert set(_declared_functions()) <= set(re.findall(r"\sT\s(qg_\w+)", out))
    dbg = ctypes.CDLL(qg.DEBUG_LIB_PATH)
    dbg.qg_debug_checks.restype = ctypes.c_int
    assert dbg.qg_debug_checks() == 1


def test_header_compiles_as_c():
    src = f'#include "{HEADER}"\nint main(void) {{ return (int)QG_OK; }}\n'
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-x", "c", "-", "-o", os.devnull],
                       input=src, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_workspace_size_contract():
    r = qg.raw
    assert r.qg_gemm_workspace_size(0, 64, 64) == 0          # empty problem
    assert r.qg_gemm_workspace_size(65, 4096, 4096) == 0     # prefill shapes use none
    small, big = r.qg_gemm_workspace_size(16, 4096, 4096), r.qg_gemm_workspace_size(64, 11008, 4096)
    assert 0 < small <= big < 64 << 20                      # modest: partial tiles + tickets


def test_status_strings_and_version():
    assert qg.raw.qg_version() >= 100
    assert qg.raw.qg_debug_checks() == 0  # the release library
    for code, name in enumerate(["QG_OK", "QG_ERR_INVALID_ARG", "QG_ERR_ALIGNMENT", "QG_ERR_UNSUPPORTED",
                                 "QG_ERR_CUDA", "QG_ERR_TIMEOUT", "QG_ERR_NO_DEVICE", "QG_ERR_DEBUG_CHECK"]):
        assert qg.raw.qg_status_string(code).decode() == name


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation happens before any launch


def _vp(x):
    return ctypes.c_void_p(x)


def test_validation_errors_without_a_device():
    r = qg.raw
    # negative size
    assert r.qg_quantize_rowwise_int8(_vp(FAKE), 64, _vp(FAKE), 64, _vp(FAKE), -1, 64, None) == qg.QG_ERR_INVALID_ARG
    # M == 0 is a no-op even without a device
    assert r.qg_quantize_rowwise_int8(_vp(FAKE), 64, _vp(FAKE), 64, _vp(FAKE), 0, 64, None) == qg.QG_OK
    assert r.qg_gemm_w8a8(None, 64, None, 64, None, None, None, None, qg.QG_F16, 64, 0, 64, 64, None, 0, None) == qg.QG_OK
    # misaligned matrix pointer / leading dimension
    assert r.qg_quantize_rowwise_int8(_vp(FAKE + 2), 64, _vp(FAKE), 64, _vp(FAKE), 4, 64, None) == qg.QG_ERR_ALIGNMENT
    assert r.qg_quantize_rowwise_int8(_vp(FAKE), 66, _vp(FAKE), 80, _vp(FAKE), 4, 64, None) == qg.QG_ERR_ALIGNMENT
    # leading dimension smaller than the row
    assert r.qg_quantize_rowwise_int8(_vp(FAKE), 32, _vp(FAKE), 64, _vp(FAKE), 4, 64, None) == qg.QG_ERR_INVALID_ARG
    # unknown output dtype, K beyond the int32 bound, null output
    assert r.qg_gemm_w8a8(_vp(FAKE), 64, _vp(FAKE), 64, _vp(FAKE), _vp(FAKE), None, _vp(FAKE), 9, 64, 4, 64, 64, None, 0, None) == qg.QG_ERR_INVALID_ARG
    assert r.qg_gemm_w8a8(_vp(FAKE), 200000, _vp(FAKE), 200000, _vp(FAKE), _vp(FAKE), None, _vp(FAKE), qg.QG_F32, 64, 4, 64, 140000, None, 0, None) == qg.QG_ERR_UNSUPPORTED
    assert r.qg_gemm_w8a8(_vp(FAKE), 64, _vp(FAKE), 64, _vp(FAKE), _vp(FAKE), None, None, qg.QG_F32, 64, 4, 64, 64, None, 0, None) == qg.QG_ERR_INVALID_ARG
    # W4A16: group other than 64, K not a multiple of the group
    assert r.qg_gemm_w4a16(_vp(FAKE), 128, _vp(FAKE), _vp(FAKE), _vp(FAKE), 128, None, _vp(FAKE), 64, 4, 64, 128, None, 0, None) == qg.QG_ERR_UNSUPPORTED
    assert r.qg_gemm_w4a16(_vp(FAKE), 128, _vp(FAKE), _vp(FAKE), _vp(FAKE), 64, None, _vp(FAKE), 64, 4, 64, 96, None, 0, None) == qg.QG_ERR_INVALID_ARG
    assert r.qg_quantize_block_asym4(_vp(FAKE), 128, _vp(FAKE), _vp(FAKE), _vp(FAKE), 8, 100, 64, None) == qg.QG_ERR_INVALID_ARG
    msg = r.qg_last_error_message().decode()
    assert "multiple" in msg


def test_tuning_and_fault_injection_arguments_are_checked():
    r = qg.raw
    assert r.qg_set_tuning(b"QG_W8A8_PAIR", 1) == qg.QG_OK
    assert r.qg_set_tuning(b"QG_PAIR_N", 0) == qg.QG_OK
    assert r.qg_set_tuning(b"QG_NO_SUCH_SWITCH", 1) == qg.QG_ERR_INVALID_ARG
    assert r.qg_set_tuning(None, 1) == qg.QG_ERR_INVALID_ARG
    assert r.qg_debug_inject_timeout(7, 1000) == qg.QG_ERR_INVALID_ARG
    assert r.qg_debug_inject_timeout(qg.QG_DEBUG_STREAM_K, 5) == qg.QG_ERR_INVALID_ARG
    assert r.qg_debug_inject_timeout(qg.QG_DEBUG_WEIGHT_ONLY, 2_000_000) == qg.QG_ERR_INVALID_ARG


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="checks the no-device path")
def test_valid_call_reports_no_device_on_a_cpu_host():
    st = qg.raw.qg_quantize_rowwise_int8(_vp(FAKE), 64, _vp(FAKE), 64, _vp(FAKE), 4, 64, None)
    assert st == qg.QG_ERR_NO_DEVICE
    with pytest.raises(ValueError):
        import torch
        qg.quantize_rowwise_int8(torch.zeros(4, 64, dtype=torch.float16))   # CPU tensor: no CPU path


def _plan(create, *args):
    h = ctypes.c_void_p()
    assert create(ctypes.byref(h), *args) == qg.QG_OK and h.value
    return h.value


def test_plan_launches_return_the_direct_calls_status():
    """A plan records its arguments; each launch runs the direct call's checks,
    so launch and direct call agree on every status, device or not."""
    r = qg.raw
    F = FAKE
    cases = [  # (plan constructor, direct call, arguments without the stream; direct: + flags where _ex)
        (r.qg_plan_quantize_rowwise_int8, r.qg_quantize_rowwise_int8, (_vp(F), 64, _vp(F), 64, _vp(F), -1, 64)),
        (r.qg_plan_quantize_rowwise_int8, r.qg_quantize_rowwise_int8, (_vp(F), 64, _vp(F), 64, _vp(F), 0, 64)),
        (r.qg_plan_quantize_rowwise_int8, r.qg_quantize_rowwise_int8, (_vp(F + 2), 64, _vp(F), 64, _vp(F), 4, 64)),
        (r.qg_plan_quantize_rowwise_int8, r.qg_quantize_rowwise_int8, (_vp(F), 32, _vp(F), 64, _vp(F), 4, 64)),
        (r.qg_plan_quantize_rowwise_int8, r.qg_quantize_rowwise_int8, (_vp(F), 64, _vp(F), 64, _vp(F), 4, 64)),
        (r.qg_plan_gemm_w8a8, r.qg_gemm_w8a8_ex,
         (_vp(F), 64, _vp(F), 64, _vp(F), _vp(F), None, _vp(F), 9, 64, 4, 64, 64, None, 0, 0)),
        (r.qg_plan_gemm_w8a8, r.qg_gemm_w8a8_ex,
         (_vp(F), 64, _vp(F), 64, _vp(F), _vp(F), None, None, qg.QG_F32, 64, 4, 64, 64, None, 0, 0)),
        (r.qg_plan_gemm_w8a8, r.qg_gemm_w8a8_ex,
         (_vp(F), 64, _vp(F), 64, _vp(F), _vp(F), None, _vp(F), qg.QG_F16, 64, 4, 64, 64, None, 0, 2)),
        (r.qg_plan_gemm_w8a8, r.qg_gemm_w8a8_ex,
         (_vp(F), 64, _vp(F), 64, _vp(F), _vp(F), None, _vp(F), qg.QG_F16, 64, 4, 64, 64, None, 0, 1)),
        (r.qg_plan_gemm_w8a16, r.qg_gemm_w8a16_ex,
         (_vp(F), 4096, _vp(F), 4096, _vp(F), None, _vp(F), 100, 16, 4096, 4096, None, 0, 0)),
        (r.qg_plan_gemm_w8a16, r.qg_gemm_w8a16_ex,
         (_vp(F), 4096, _vp(F), 4096, _vp(F), None, _vp(F), 4096, 16, 4096, 4096, None, 0, 1)),
        (r.qg_plan_gemm_w4a16, r.qg_gemm_w4a16_ex,
         (_vp(F), 128, _vp(F), _vp(F), _vp(F), 128, None, _vp(F), 64, 4, 64, 128, None, 0, 0)),
        (r.qg_plan_gemm_w4a16, r.qg_gemm_w4a16_ex,
         (_vp(F), 128, _vp(F), _vp(F), _vp(F), 64, None, _vp(F), 64, 4, 64, 96, None, 0, 0)),
        (r.qg_plan_gemm_w4a16, r.qg_gemm_w4a16_ex,
         (_vp(F), 128, _vp(F), _vp(F), _vp(F), 64, None, _vp(F), 64, 4, 64, 128, None, 0, 1)),
    ]
    seen = set()
    for create, direct, args in cases:
        h = _plan(create, *args)
        try:
            for _ in range(2):  # a launch leaves the plan unchanged
                st = r.qg_plan_launch(h, None)
                assert st == direct(*args, None), (direct.__name__, args)
            seen.add(st)
        finally:
            r.qg_plan_destroy(h)
    assert {qg.QG_OK, qg.QG_ERR_INVALID_ARG, qg.QG_ERR_ALIGNMENT, qg.QG_ERR_UNSUPPORTED} <= seen


def test_plan_null_handling():
    r = qg.raw
    assert r.qg_plan_launch(None, None) == qg.QG_ERR_INVALID_ARG
    r.qg_plan_destroy(None)  # a no-op
    assert r.qg_plan_gemm_w8a16(None, _vp(FAKE), 64, _vp(FAKE), 64, _vp(FAKE), None, _vp(FAKE), 64, 4, 64, 64,
                                None, 0, 0) == qg.QG_ERR_INVALID_ARG
    assert "plan" in r.qg_last_error_message().decode()
    with pytest.raises(ValueError):  # the binding: plans keep their workspace, so no per-stream 'auto' one
        qg._plan_workspace("auto")
