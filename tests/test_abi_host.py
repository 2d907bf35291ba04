"""CPU-only checks of the C ABI: the library loads, exports every entry point that
include/w4.h declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import pytest

from bit_gemm_wise_b200 import w4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "w4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(w4\w*|fp8_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(w4.LIB_PATH):
        from bit_gemm_wise_b200 import build
        build.build()
    return w4.lib()


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert {"w4_quantize", "w4a16_gemv", "w4a8_gemm", "fp8_row_quant", "w4_prepack",
            "w4a8_grouped_gemm", "w4_device_status"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    bound = {n for n, _, _ in w4.SIGNATURES}
    assert set(names) <= bound


def test_status_strings_and_version(lib):
    assert w4.w4_version() >= 100
    for code, name in w4.STATUS.items():
        s = w4.w4_status_str(code)
        assert s and s != "unknown status", (code, name)
    assert w4.w4_status_str(999) == "unknown status"


def test_prepack_bytes(lib):
    # GEMV layout: codes of N padded to 8 and K to 128, plus 4 bytes per (row, group)
    assert w4.w4_prepack_bytes(4096, 4096, 128, w4.W4_LAYOUT_GEMV) == 4096 * 4096 // 2 + 4096 * 32 * 4
    assert w4.w4_prepack_bytes(1536, 576, 32, w4.W4_LAYOUT_GEMV) == 1536 * 640 // 2 + 1536 * 20 * 4
    # GEMM layout: rows and K padded to 128; codes, scales of the padded groups, and the
    # zero-point operand with 3 * 90 real groups rounded up to 288 bf16 columns
    assert w4.w4_prepack_bytes(2880, 2880, 32, w4.W4_LAYOUT_GEMM) == \
        2944 * 2944 // 2 + 92 * 2944 * 4 + 2944 * 288 * 2
    assert w4.w4_prepack_bytes(3840, 15360, 128, w4.W4_LAYOUT_GEMM) == \
        3840 * 15360 // 2 + 120 * 3840 * 4 + 3840 * 384 * 2
    for bad in [(0, 4096, 128), (16, 100, 32), (16, 4096, 48), (16, 96, 64)]:
        assert w4.w4_prepack_bytes(*bad, w4.W4_LAYOUT_GEMV) == 0
    assert w4.w4_prepack_bytes(16, 4096, 128, 7) == 0


def test_gsum_op_cols(lib):
    assert w4.w4a8_gsum_op_cols(2880, 32) == 288
    assert w4.w4a8_gsum_op_cols(4096, 128) == 96
    assert w4.w4a8_gsum_op_cols(15360, 128) == 384
    assert w4.w4a8_gsum_op_cols(3840, 128) == 96
    assert w4.w4a8_gsum_op_cols(160, 32) == 32
    for bad in [(96, 64), (128, 48), (0, 32)]:
        assert w4.w4a8_gsum_op_cols(*bad) == 0


FAKE = 0x1000  # 16-byte aligned non-null address; never dereferenced (calls fail validation)


def rc(fn, *args):
    return getattr(w4.lib(), fn)(*args)


def test_host_validation_rejects_before_launch(lib):
    grid = (ctypes.c_float * 2)(1.0, 0.9)
    gp = ctypes.cast(grid, ctypes.c_void_p)
    # null pointers
    assert rc("w4_quantize", None, 16, 128, 128, 1, gp, 2, FAKE, FAKE, FAKE, None, None) == 1
    # zeros required for asym, forbidden for sym
    assert rc("w4_quantize", FAKE, 16, 128, 128, 1, gp, 2, FAKE, FAKE, None, None, None) == 1
    assert rc("w4_quantize", FAKE, 16, 128, 128, 0, gp, 2, FAKE, FAKE, FAKE, None, None) == 5
    # shapes and groups
    assert rc("w4_quantize", FAKE, 0, 128, 128, 1, gp, 2, FAKE, FAKE, FAKE, None, None) == 2
    assert rc("w4_quantize", FAKE, 16, 100, 32, 1, gp, 2, FAKE, FAKE, FAKE, None, None) == 2
    assert rc("w4_quantize", FAKE, 16, 96, 64, 1, gp, 2, FAKE, FAKE, FAKE, None, None) == 3
    assert rc("w4_quantize", FAKE, 16, 128, 48, 1, gp, 2, FAKE, FAKE, FAKE, None, None) == 3
    # misaligned pointer
    assert rc("w4_quantize", FAKE + 2, 16, 128, 128, 1, gp, 2, FAKE, FAKE, FAKE, None, None) == 4
    # clip grid: first ratio must be 1.0, all in (0, 1], finite, at most 64
    bad = (ctypes.c_float * 2)(0.9, 1.0)
    assert rc("w4_quantize", FAKE, 16, 128, 128, 1, ctypes.cast(bad, ctypes.c_void_p), 2, FAKE, FAKE, FAKE,
              None, None) == 5
    nan = (ctypes.c_float * 2)(1.0, float("nan"))
    assert rc("w4_quantize", FAKE, 16, 128, 128, 1, ctypes.cast(nan, ctypes.c_void_p), 2, FAKE, FAKE, FAKE,
              None, None) == 5
    assert rc("w4_quantize", FAKE, 16, 128, 128, 1, gp, 0, FAKE, FAKE, FAKE, None, None) == 5
    assert rc("w4_quantize", FAKE, 16, 128, 128, 1, gp, 65, FAKE, FAKE, FAKE, None, None) == 5
    # row quant
    assert rc("fp8_row_quant", None, 4, 64, 32, FAKE, FAKE, None, None, None) == 1
    assert rc("fp8_row_quant", FAKE, 4, 72, 32, FAKE, FAKE, None, None, None) == 2
    assert rc("fp8_row_quant", FAKE, 4, 96, 64, FAKE, FAKE, FAKE, None, None) == 3
    assert rc("fp8_row_quant", FAKE, 4, 96, 64, FAKE, FAKE, None, FAKE, None) == 3
    assert rc("fp8_row_quant", FAKE, 4, 128, 64, FAKE, FAKE, None, FAKE + 4, None) == 4
    # gemv: M range, mode, out flag
    assert rc("w4a16_gemv", FAKE, 17, FAKE, 16, 128, 128, 1, FAKE, 0, FAKE, 1 << 20, None) == 2
    assert rc("w4a16_gemv", FAKE, 1, FAKE, 16, 128, 128, 3, FAKE, 0, FAKE, 1 << 20, None) == 5
    assert rc("w4a16_gemv", FAKE, 1, FAKE, 16, 128, 128, 1, FAKE, 4, FAKE, 1 << 20, None) == 5
    assert rc("w4a16_gemv", FAKE, 1, FAKE, 16, 128, 128, 1, FAKE, 0, FAKE + 8, 1 << 20, None) == 4
    # gemm: the group-sum operand is required, K >= 128
    assert rc("w4a8_gemm", FAKE, FAKE, None, 4, FAKE, 16, 128, 128, 1, FAKE, 0, None) == 1
    assert rc("w4a8_gemm", FAKE, FAKE, FAKE, 4, FAKE, 16, 96, 32, 1, FAKE, 0, None) == 2
    # grouped gemm: expert count range
    assert rc("w4a8_grouped_gemm", FAKE, FAKE, FAKE, FAKE, 0, 16, FAKE, 16, 128, 128, 1, FAKE, None) == 2
    # prepack
    assert rc("w4_prepack", FAKE, FAKE, None, 16, 128, 128, 1, 0, FAKE, None) == 1
    assert rc("w4_prepack", FAKE, FAKE, None, 16, 128, 128, 0, 9, FAKE, None) == 5
    # device status needs an out pointer
    assert rc("w4_device_status", None, None) == 1
