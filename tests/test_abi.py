"""The C-ABI library builds, loads and exports every entry point that
include/lightning.h declares; host-side argument validation answers without a
GPU (no compute call is made: validation fails before any CUDA call)."""
import ctypes
import os
import re

import pytest

import linear_attention_13_b200 as la
from linear_attention_13_b200 import build as labuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_entry_points():
    text = open(os.path.join(ROOT, "include", "lightning.h")).read()
    return sorted(set(re.findall(r"^(?:int|const char\*)\s+(la_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def lib():
    labuild.build()
    return la.load_library()


def test_header_declares_expected_entry_points():
    names = _declared_entry_points()
    for n in ("la_prefill", "la_prefill_varlen", "la_decode_step", "la_status_string",
              "la_get_last_error"):
        assert n in names
    assert set(names) == set(la.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for n in _declared_entry_points():
        assert hasattr(lib, n), n
        assert isinstance(getattr(lib, n), ctypes._CFuncPtr)


def test_library_is_built_for_sm100a():
    # the build compiles for sm_100a only (the GPU test reads the loaded code
    # object's version through la_binary_version)
    flags = labuild.NVCC_FLAGS
    i = flags.index("-gencode")
    assert flags[i + 1] == "arch=compute_100a,code=sm_100a"
    assert flags.count("-gencode") == 1 and not any("-arch" == f for f in flags)


def test_debug_allocation_failures_validate_their_count(lib):
    assert la.la_debug_fail_allocations(-1) == la.LA_ERR_INVALID_ARG
    assert la.la_debug_fail_allocations(0) == la.LA_OK


def test_status_strings(lib):
    assert la.status_string(la.LA_OK) == "LA_OK"
    assert la.status_string(la.LA_ERR_BAD_SEQLENS) == "LA_ERR_BAD_SEQLENS"
    assert la.status_string(la.LA_ERR_BAD_SLOT) == "LA_ERR_BAD_SLOT"
    assert la.status_string(12345) == "LA_UNKNOWN_STATUS"


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++11")])
def test_header_compiles_as_plain_c_and_cpp(tmp_path, compiler, std):
    # the boundary is a C ABI: the header alone must compile in C and C++
    src = tmp_path / ("use.c" if compiler == "gcc" else "use.cpp")
    src.write_text('#include "lightning.h"\n'
                   "int main(void) {\n"
                   "    la_dtype dt = LA_BF16;\n"
                   "    int (*f)(const void*, const void*, const void*, void*, float*, int, int, int,\n"
                   "             int, int, la_dtype, void*) = la_prefill;\n"
                   "    return (f != 0 && dt == LA_BF16 && LA_ERR_BAD_SLOT < 0) ? 0 : 1;\n"
                   "}\n")
    import subprocess
    r = subprocess.run([compiler, std, "-Wall", "-Werror", "-pedantic", "-fsyntax-only",
                        "-I", os.path.join(ROOT, "include"), str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


FAKE = 0x100000  # 16-byte aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("args,expect", [
    ((None, FAKE, FAKE, FAKE, None, 1, 1, 16, 128, 128, la.LA_BF16, None), la.LA_ERR_INVALID_ARG),
    ((FAKE + 2, FAKE, FAKE, FAKE, None, 1, 1, 16, 128, 128, la.LA_BF16, None), la.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, None, 0, 1, 16, 128, 128, la.LA_BF16, None), la.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 1, 0, 128, 128, la.LA_BF16, None), la.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 96, 128, la.LA_BF16, None), la.LA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 64, 128, la.LA_BF16, None), la.LA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 128, 32, la.LA_BF16, None), la.LA_ERR_UNSUPPORTED),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 128, 0, la.LA_F32, None), la.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, None, 1, 1, 16, 128, 64, 7, None), la.LA_ERR_INVALID_ARG),
    ((FAKE, FAKE, FAKE, FAKE, FAKE + 4, 1, 1, 16, 128, 64, la.LA_F32, None), la.LA_ERR_INVALID_ARG),
])
def test_prefill_argument_validation(lib, args, expect):
    assert la.la_prefill(*args) == expect


def test_varlen_and_decode_argument_validation(lib):
    assert la.la_prefill_varlen(FAKE, FAKE, FAKE, FAKE, None, None, 1, 16, 1, 128, 128,
                                la.LA_BF16, None) == la.LA_ERR_INVALID_ARG
    assert la.la_prefill_varlen(FAKE, FAKE, FAKE, FAKE, None, FAKE + 2, 1, 16, 1, 128, 128,
                                la.LA_BF16, None) == la.LA_ERR_INVALID_ARG
    assert la.la_prefill_varlen(FAKE, FAKE, FAKE, FAKE, None, FAKE, 0, 16, 1, 128, 128,
                                la.LA_BF16, None) == la.LA_ERR_INVALID_ARG
    assert la.la_decode_step(FAKE, FAKE, FAKE, None, FAKE, 1, 1, 128, la.LA_BF16,
                             None) == la.LA_ERR_INVALID_ARG
    assert la.la_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 32, la.LA_BF16,
                             None) == la.LA_ERR_UNSUPPORTED
    assert la.la_decode_step(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 1, 128, la.LA_BF16,
                             None) == la.LA_ERR_INVALID_ARG


def test_slot_decode_and_8bit_state_argument_validation(lib):
    I, U = la.LA_ERR_INVALID_ARG, la.LA_ERR_UNSUPPORTED
    # slot pool: misaligned slot array, empty pool, no slots with a pool smaller than B
    assert la.la_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE + 2, 4, FAKE, 2, 1, 128,
                                   la.LA_BF16, None) == I
    assert la.la_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, 2, 1, 128,
                                   la.LA_BF16, None) == I
    assert la.la_decode_step_slots(FAKE, FAKE, FAKE, FAKE, None, 1, FAKE, 2, 1, 128,
                                   la.LA_BF16, None) == I
    assert la.la_decode_step_slots(FAKE, FAKE, FAKE, None, FAKE, 4, FAKE, 2, 1, 128,
                                   la.LA_BF16, None) == I
    assert la.la_decode_step_slots(FAKE, FAKE, FAKE, FAKE, FAKE, 4, FAKE, 2, 1, 96,
                                   la.LA_BF16, None) == U
    # 8-bit state: missing or misaligned codes / scales
    assert la.la_decode_step_q8(FAKE, FAKE, FAKE, None, FAKE, None, 2, FAKE, 2, 1, 128,
                                la.LA_BF16, None) == I
    assert la.la_decode_step_q8(FAKE, FAKE, FAKE, FAKE, FAKE + 4, None, 2, FAKE, 2, 1, 128,
                                la.LA_BF16, None) == I
    assert la.la_decode_step_q8(FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, FAKE, 2, 1, 128,
                                la.LA_BF16, None) == I
    assert la.la_state_quantize_q8(FAKE, FAKE, FAKE, 0, 128, None) == I
    assert la.la_state_quantize_q8(FAKE, FAKE, FAKE, 1, 96, None) == U
    assert la.la_state_dequantize_q8(FAKE, None, FAKE, 1, 128, None) == I
    assert la.la_state_dequantize_q8(FAKE, FAKE, FAKE, 1, 32, None) == U


def test_backward_and_sequence_parallel_argument_validation(lib):
    I = la.LA_ERR_INVALID_ARG
    assert la.la_prefill_backward(FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 1, 16, 128, 128,
                                  la.LA_BF16, None) == I
    assert la.la_prefill_backward(FAKE, FAKE, FAKE, FAKE, FAKE + 2, FAKE, FAKE, 1, 1, 16, 128,
                                  128, la.LA_BF16, None) == I
    assert la.la_prefill_backward(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 0, 128, 128,
                                  la.LA_BF16, None) == I
    assert la.la_state_increment(None, FAKE, FAKE, 1, 1, 16, 128, la.LA_BF16, None) == I
    assert la.la_state_increment(FAKE, FAKE, FAKE, 1, 1, 16, 64, la.LA_BF16,
                                 None) == la.LA_ERR_UNSUPPORTED


@pytest.mark.parametrize("flags", [
    la.LA_FLAG_SPLIT_V | la.LA_FLAG_THREE_PASS,
    la.LA_FLAG_SPLIT_V | la.LA_FLAG_FUSED,
    la.LA_FLAG_SPLIT_V | la.LA_FLAG_NO_SPLIT_V,
    la.LA_FLAG_THREE_PASS | la.LA_FLAG_FUSED,
    64,
])
def test_varlen_schedule_flag_validation(lib, flags):
    # rejected before anything touches the device
    assert la.la_prefill_varlen_ex(FAKE, FAKE, FAKE, FAKE, None, FAKE, 1, 16, 1, 128, 128,
                                   la.LA_BF16, None, 0, flags) == la.LA_ERR_INVALID_ARG


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        la.load_library(str(tmp_path / "nope.so"))
