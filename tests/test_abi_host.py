"""CPU-only checks of the C ABI: the library loads, exports every entry point that
include/w4.h declares, and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import numpy as np
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
    # one record per row: K/2 code bytes, then K/g scale words padded to 16 bytes
    assert w4.w4_prepack_bytes(4096, 4096, 128, w4.W4_LAYOUT_GEMV) == 4096 * (4096 // 2 + 32 * 4)
    assert w4.w4_prepack_bytes(1536, 576, 32, w4.W4_LAYOUT_GEMV) == 1536 * (576 // 2 + 80)
    # GEMM layout: rows and K padded to 128; codes, scales of the padded groups, and the
    # zero-point operand with 3 * 90 real groups rounded up to 288 bf16 columns
    assert w4.w4_prepack_bytes(2880, 2880, 32, w4.W4_LAYOUT_GEMM) == \
        2944 * 2944 // 2 + 92 * 2944 * 4 + 2944 * 288 * 2
    assert w4.w4_prepack_bytes(3840, 15360, 128, w4.W4_LAYOUT_GEMM) == \
        3840 * 15360 // 2 + 120 * 3840 * 4 + 3840 * 384 * 2
    for bad in [(0, 4096, 128), (16, 100, 32), (16, 4096, 48), (16, 96, 64)]:
        assert w4.w4_prepack_bytes(*bad, w4.W4_LAYOUT_GEMV) == 0
    assert w4.w4_prepack_bytes(16, 4096, 128, 7) == 0
    # tensor-core W4A16 layout: units of 128 rows x max(128, g) k, each KS/2 code bytes per row
    # and 4 bytes per (row, group); rows padded to 128, K to the unit's k
    assert w4.w4_prepack_bytes(4096, 4096, 128, w4.W4_LAYOUT_TC) == 32 * 32 * (128 * 64 + 512)
    assert w4.w4_prepack_bytes(77, 320, 32, w4.W4_LAYOUT_TC) == 1 * 3 * (128 * 64 + 4 * 512)
    assert w4.w4_prepack_bytes(200, 768, 256, w4.W4_LAYOUT_TC) == 2 * 3 * (128 * 128 + 512)


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
    # row quant: codes or their fp16 copy (or both) required
    assert rc("fp8_row_quant", None, 4, 64, 32, FAKE, FAKE, None, None, None, None) == 1
    assert rc("fp8_row_quant", FAKE, 4, 64, 32, None, FAKE, None, None, None, None) == 1
    assert rc("fp8_row_quant", FAKE, 4, 72, 32, FAKE, FAKE, None, None, None, None) == 2
    assert rc("fp8_row_quant", FAKE, 4, 96, 64, FAKE, FAKE, FAKE, None, None, None) == 3
    assert rc("fp8_row_quant", FAKE, 4, 96, 64, FAKE, FAKE, None, FAKE, None, None) == 3
    assert rc("fp8_row_quant", FAKE, 4, 128, 64, FAKE, FAKE, None, FAKE + 4, None, None) == 4
    assert rc("fp8_row_quant", FAKE, 4, 128, 64, None, FAKE, None, None, FAKE + 8, None) == 4
    # gemv: M range, mode, out flag
    assert rc("w4a16_gemv", FAKE, 17, FAKE, 16, 128, 128, 1, FAKE, 0, FAKE, 1 << 20, None) == 2
    assert rc("w4a16_gemv", FAKE, 1, FAKE, 16, 128, 128, 3, FAKE, 0, FAKE, 1 << 20, None) == 5
    assert rc("w4a16_gemv", FAKE, 1, FAKE, 16, 128, 128, 1, FAKE, 4, FAKE, 1 << 20, None) == 5
    assert rc("w4a16_gemv", FAKE, 1, FAKE, 16, 128, 128, 1, FAKE, 0, FAKE + 8, 1 << 20, None) == 4
    # gemv naming the next GEMV's weights: a byte count needs a pointer, the pointer 16-byte
    # alignment; the other checks are w4a16_gemv's
    assert rc("w4a16_gemv_prefetch_next", FAKE, 1, FAKE, 16, 128, 128, 1, FAKE, 0, None, 0, None, 4096, None) == 1
    assert rc("w4a16_gemv_prefetch_next", FAKE, 1, FAKE, 16, 128, 128, 1, FAKE, 0, None, 0, FAKE + 8, 4096,
              None) == 4
    assert rc("w4a16_gemv_prefetch_next", FAKE, 17, FAKE, 16, 128, 128, 1, FAKE, 0, None, 0, FAKE, 4096, None) == 2
    assert rc("w4a16_gemv_prefetch_next", FAKE, 1, FAKE, 16, 128, 128, 3, FAKE, 0, None, 0, FAKE, 4096, None) == 5
    # tensor-core w4a16: M in 1..16, a workspace of the queried size, flags as the GEMV's
    tws = lib.w4a16_gemm_tc_workspace_bytes(4096, 4096, 128)
    assert tws > 0 and tws % 16 == 0
    assert lib.w4a16_gemm_tc_workspace_bytes(4096, 100, 128) == 0
    assert rc("w4a16_gemm_tc", None, 4, FAKE, 4096, 4096, 128, 1, FAKE, 0, FAKE, tws, None) == 1
    assert rc("w4a16_gemm_tc", FAKE, 17, FAKE, 4096, 4096, 128, 1, FAKE, 0, FAKE, tws, None) == 2
    assert rc("w4a16_gemm_tc", FAKE, 0, FAKE, 4096, 4096, 128, 1, FAKE, 0, FAKE, tws, None) == 2
    assert rc("w4a16_gemm_tc", FAKE, 4, FAKE, 4096, 4096, 48, 1, FAKE, 0, FAKE, tws, None) == 3
    assert rc("w4a16_gemm_tc", FAKE, 4, FAKE, 4096, 4096, 128, 3, FAKE, 0, FAKE, tws, None) == 5
    assert rc("w4a16_gemm_tc", FAKE, 4, FAKE, 4096, 4096, 128, 1, FAKE, 8, FAKE, tws, None) == 5
    assert rc("w4a16_gemm_tc", FAKE, 4, FAKE, 4096, 4096, 128, 1, FAKE + 2, 0, FAKE, tws, None) == 4
    assert rc("w4a16_gemm_tc", FAKE, 4, FAKE, 4096, 4096, 128, 1, FAKE, 0, None, 0, None) == 10
    assert rc("w4a16_gemm_tc", FAKE, 4, FAKE, 4096, 4096, 128, 1, FAKE, 0, FAKE, tws - 16, None) == 10
    # gemm: groups 64/128 need the codes and the group-sum operand, groups 32/256 the fp16
    # copy of the activations; K >= 128
    assert rc("w4a8_gemm", FAKE, None, FAKE, None, 4, FAKE, 16, 128, 128, 1, FAKE, 0, None, 0, None) == 1
    assert rc("w4a8_gemm", None, FAKE, FAKE, FAKE, 4, FAKE, 16, 128, 128, 1, FAKE, 0, None, 0, None) == 1
    assert rc("w4a8_gemm", FAKE, None, FAKE, FAKE, 4, FAKE, 16, 128, 32, 1, FAKE, 0, None, 0, None) == 1
    assert rc("w4a8_gemm", FAKE, FAKE, FAKE, FAKE, 4, FAKE, 16, 96, 32, 1, FAKE, 0, None, 0, None) == 2
    assert rc("w4a8_gemm", FAKE, None, FAKE, FAKE, 4, FAKE, 16, 128, 128, 1, FAKE, 0, FAKE + 8, 1 << 20, None) == 4
    assert rc("w4a8_gemm", None, FAKE + 4, FAKE, None, 4, FAKE, 16, 256, 256, 1, FAKE, 0, None, 0, None) == 4
    # grouped gemm: expert count range
    assert rc("w4a8_grouped_gemm", FAKE, None, FAKE, FAKE, FAKE, 0, 16, FAKE, 16, 128, 128, 1, FAKE, None) == 2
    # prepack
    assert rc("w4_prepack", FAKE, FAKE, None, 16, 128, 128, 1, 0, FAKE, None) == 1
    assert rc("w4_prepack", FAKE, FAKE, None, 16, 128, 128, 0, 9, FAKE, None) == 5
    # moe route: expert and top-k ranges, workspace size
    ws = lib.w4_moe_route_workspace_bytes(100, 32)
    assert ws == 4 * 32 * 4  # ceil(100 / 32) blocks of 32 expert counts
    assert lib.w4_moe_route_workspace_bytes(0, 32) == 0
    assert rc("w4_moe_route", FAKE, 100, 32, 4, FAKE, FAKE, FAKE, FAKE, FAKE, None, ws, None) == 1
    assert rc("w4_moe_route", FAKE, 100, 1025, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 2
    assert rc("w4_moe_route", FAKE, 100, 32, 9, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == 2
    assert rc("w4_moe_route", FAKE, 100, 4, 5, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == 2
    assert rc("w4_moe_route", FAKE, 100, 32, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws - 4, None) == 10
    assert rc("w4_moe_route", FAKE + 2, 100, 32, 4, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None) == 4
    # device status needs an out pointer
    assert rc("w4_device_status", None, None) == 1


def test_gemm_rowquant_layout_and_validation(lib):
    """The one-launch row quant + GEMM: workspace regions 256-byte aligned, in order, sized
    for M x K codes, M scales and the group-sum operand; host checks before any launch."""
    for M, N, K, g in [(4096, 15360, 3840, 128), (4096, 3840, 15360, 128), (7, 77, 192, 64), (1, 128, 128, 128)]:
        lay = w4.w4a8_gemm_rowquant_layout(M, N, K, g)
        cols = w4.w4a8_gsum_op_cols(K, g)
        assert all(lay[k] % 256 == 0 for k in lay)
        assert lay["X_e4m3"] + M * K <= lay["row_scale"]
        assert lay["row_scale"] + 4 * M <= lay["gsum_op"]
        assert lay["gsum_op"] + 2 * M * cols <= lay["bytes"]
        assert lay["bytes"] == w4.w4a8_gemm_rowquant_workspace_bytes(M, N, K, g)
        # the split tiles' partials and counters come first, then one row counter per token tile
        sched = w4.w4a8_gemm_schedule(M, N, K, g, 148)
        assert lay["X_e4m3"] >= sched["workspace_bytes"] + 4 * ((M + 255) // 256)
    # groups of 32 and 256 (the split-weight path) are not offered
    assert lib.w4a8_gemm_rowquant_workspace_bytes(4096, 4096, 4096, 32) == 0
    assert lib.w4a8_gemm_rowquant_workspace_bytes(4096, 4096, 4096, 256) == 0
    ws = w4.w4a8_gemm_rowquant_workspace_bytes(64, 256, 512, 128)
    assert rc("w4a8_gemm_rowquant", None, 64, FAKE, 256, 512, 128, 1, FAKE, 0, FAKE, ws, None) == 1
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 512, 128, 1, FAKE, 0, None, ws, None) == 1
    assert rc("w4a8_gemm_rowquant", FAKE, 0, FAKE, 256, 512, 128, 1, FAKE, 0, FAKE, ws, None) == 2
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 96, 32, 1, FAKE, 0, FAKE, ws, None) == 2
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 512, 48, 1, FAKE, 0, FAKE, ws, None) == 3
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 512, 32, 1, FAKE, 0, FAKE, ws, None) == 6
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 512, 128, 3, FAKE, 0, FAKE, ws, None) == 5
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 512, 128, 1, FAKE, 2, FAKE, ws, None) == 5
    assert rc("w4a8_gemm_rowquant", FAKE + 8, 64, FAKE, 256, 512, 128, 1, FAKE, 0, FAKE, ws, None) == 4
    assert rc("w4a8_gemm_rowquant", FAKE, 64, FAKE, 256, 512, 128, 1, FAKE, 0, FAKE + 16, ws, None) == 4
    with pytest.raises(w4.W4Error):
        w4.w4a8_gemm_rowquant_layout(64, 256, 512, 32)


# ------------------------------------------------------------------ W4A8 GEMM work split

def test_gemm_schedule_of_the_prefill_shapes(lib):
    # 4096 tokens x 15360 -> 3840: 16 x 30 = 480 tiles on 148 SMs, three full waves; the last
    # 36 tiles (120 k-blocks each) are split over all 148 blocks
    s = w4.w4a8_gemm_schedule(4096, 3840, 15360, 128, 148)
    assert (s["tiles"], s["whole_tiles"], s["split_tiles"], s["split_blocks"], s["grid"], s["k_blocks"]) == \
        (480, 444, 36, 148, 148, 120)
    assert s["workspace_bytes"] == 2 * 148 * 128 * 256 * 4 + 36 * 8 * 4
    # 3840 -> 15360: 1920 tiles, the last wave has 144 of 148: left whole
    s = w4.w4a8_gemm_schedule(4096, 15360, 3840, 128, 148)
    assert (s["whole_tiles"], s["split_tiles"], s["grid"], s["workspace_bytes"]) == (1920, 0, 148, 0)
    # two long tiles: 8 parts each (at most 8 contributors per tile), 15 k-blocks per part
    s = w4.w4a8_gemm_schedule(256, 256, 15360, 128, 148)
    assert (s["whole_tiles"], s["split_tiles"], s["split_blocks"], s["grid"]) == (0, 2, 16, 16)
    # ragged K (2880 -> 23 k-blocks, the last one partial): 4 tiles over 8 blocks (2 per tile)
    s = w4.w4a8_gemm_schedule(300, 256, 2880, 64, 148)
    assert (s["tiles"], s["split_tiles"], s["split_blocks"], s["k_blocks"]) == (4, 4, 8, 23)
    # groups of 32 take the split-weight fp16 kernel, which keeps every tile whole
    s = w4.w4a8_gemm_schedule(300, 256, 2880, 32, 148)
    assert (s["split_tiles"], s["workspace_bytes"], s["grid"]) == (0, 0, 4)
    assert w4.w4a8_gemm_workspace_bytes(300, 256, 2880, 32) == 0
    # short K: too few k-blocks per block to split
    s = w4.w4a8_gemm_schedule(1000, 130, 640, 128, 148)
    assert (s["split_tiles"], s["grid"], s["workspace_bytes"]) == (0, 8, 0)
    with pytest.raises(w4.W4Error):
        w4.w4a8_gemm_schedule(4096, 3840, 15360, 48, 148)


@pytest.mark.parametrize("R,KT,PS", [(36, 120, 148), (2, 120, 16), (4, 23, 11), (12, 90, 96), (1, 9, 1),
                                     (7, 5, 7), (3, 1000, 148), (100, 13, 131), (147, 8, 148)])
def test_gemm_split_segments_cover_each_k_block_once(lib, R, KT, PS):
    """Every k-block of every split tile belongs to exactly one block's segment; a block has at
    most two segments, stored in slots 2c and 2c+1; each tile has one segment that ends it (and
    adds the zero-point term); every segment names the same contiguous contributor range."""
    cover = {}
    contributors = {}
    slots = set()
    for c in range(PS):
        for s in range(3):
            seg = w4.w4a8_gemm_split_segment(R, KT, PS, c, s)
            if s == 2:
                assert seg is None
            if seg is None:
                continue
            i, kb0, kb1, c0, c1, slot = seg
            assert 0 <= i < R and 0 <= kb0 < kb1 <= KT
            assert slot == 2 * c + s and slot not in slots
            slots.add(slot)
            assert c0 <= c <= c1 < PS
            assert contributors.setdefault(i, (c0, c1)) == (c0, c1)
            for kb in range(kb0, kb1):
                assert (i, kb) not in cover
                cover[(i, kb)] = c
    assert len(cover) == R * KT
    for i in range(R):
        owners = sorted({cover[(i, kb)] for kb in range(KT)})
        assert owners == list(range(contributors[i][0], contributors[i][1] + 1))
        assert cover[(i, 0)] == contributors[i][0] and cover[(i, KT - 1)] == contributors[i][1]


def test_gemm_split_segments_random(lib):
    rng = __import__("random").Random(3)
    for _ in range(40):
        PS = rng.randint(1, 300)
        R = rng.randint(1, PS)
        KT = rng.randint(-(-PS // R), 200)  # every block gets at least one k-block
        test_gemm_split_segments_cover_each_k_block_once(lib, R, KT, PS)


def test_gemm_split_segment_arguments(lib):
    with pytest.raises(w4.W4Error):
        w4.w4a8_gemm_split_segment(10, 8, 9, 0, 0)  # fewer blocks than tiles
    with pytest.raises(w4.W4Error):
        w4.w4a8_gemm_split_segment(2, 8, 16, 16, 0)  # block out of range
    with pytest.raises(w4.W4Error):
        w4.w4a8_gemm_split_segment(1, 9, 12, 0, 0)  # more blocks than k-blocks: empty ranges


# ------------------------------------------------------------------ W4A16 GEMV work split

@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)])
def test_gemv_decode_shapes_one_block_per_sm(lib, K, N):
    """M = 1 on 148 SMs: whole rows per block (no K split, no workspace), N spread over at
    most 148 blocks in contiguous runs that differ by at most one row's share."""
    s = w4.w4a16_gemv_schedule(1, N, K, 128, 148)
    assert s["rows_per_sweep"] == 1 and s["sweeps"] == 1 and s["k_parts"] == 1
    assert s["workspace_bytes"] == 0
    assert s["rows_per_block"] == -(-N // 148)
    assert s["row_blocks"] == -(-N // s["rows_per_block"]) <= 148
    assert s["stages"] >= 3 and s["smem_bytes"] <= 227 * 1024


def test_gemv_activation_rows_per_sweep(lib):
    # up to 4 activation rows ride along in registers while K/32 slices fit the block
    s = w4.w4a16_gemv_schedule(16, 4096, 14336, 128, 148)
    assert s["rows_per_sweep"] == 4 and s["sweeps"] == 4 and s["k_parts"] == 1
    s = w4.w4a16_gemv_schedule(3, 4096, 4096, 128, 148)
    assert s["rows_per_sweep"] == 4 and s["sweeps"] == 1
    assert w4.w4a16_gemv_schedule(2, 4096, 4096, 128, 148)["rows_per_sweep"] == 2
    # longer rows hold fewer activation rows per sweep
    s = w4.w4a16_gemv_schedule(4, 8192, 28672, 128, 148)
    assert s["rows_per_sweep"] == 2 and s["sweeps"] == 2 and s["k_parts"] == 1
    with pytest.raises(w4.W4Error):
        w4.w4a16_gemv_schedule(17, 4096, 4096, 128, 148)


def test_gemv_long_rows_split_along_k(lib):
    """A row whose slices (128 k each at M = 1) exceed one block's 448 threads, or whose
    activation planes (3 bytes per k) and two ring stages exceed its shared memory, is split
    into parts of a multiple of 512 k; the parts' sums go through the workspace."""
    s = w4.w4a16_gemv_schedule(1, 512, 65536, 128, 148)
    assert s["k_parts"] == 2 and s["workspace_bytes"] > 0
    assert w4.w4a16_gemv_workspace_bytes(512, 65536, 128) >= s["workspace_bytes"]
    assert w4.w4a16_gemv_schedule(1, 512, 32768, 128, 148)["k_parts"] == 1
    assert w4.w4a16_gemv_workspace_bytes(4096, 14336, 128) == 0


def test_gemm_schedule_invariants_over_many_shapes(lib):
    """For any shape and SM count: the grid fits the SMs, whole and split tiles add up, a
    split wave is partial, its blocks number at least the split tiles (so a block's range
    touches at most two tiles) and at most the SMs, and the workspace holds 2 slots per
    split block plus 8 counters per split tile."""
    rng = __import__("random").Random(7)
    for _ in range(400):
        M = rng.choice([1, 7, 256, 300, 1000, 4096, 9000])
        N = rng.choice([128, 200, 1536, 3840, 4096, 15360])
        K = rng.choice([128, 256, 576, 2880, 3840, 8192, 15360])
        g = rng.choice([g for g in (32, 64, 128, 256) if K % g == 0])
        sms = rng.choice([1, 2, 8, 132, 148, 160])
        s = w4.w4a8_gemm_schedule(M, N, K, g, sms)
        assert 1 <= s["grid"] <= sms
        assert s["whole_tiles"] + s["split_tiles"] == s["tiles"] == -(-M // 256) * -(-N // 128)
        if s["split_tiles"]:
            assert s["split_tiles"] < sms and s["split_tiles"] <= s["split_blocks"] <= sms
            assert s["whole_tiles"] % sms == 0
            assert s["split_tiles"] * s["k_blocks"] >= 8 * s["split_blocks"]  # >= 8 k-blocks per block
            assert s["workspace_bytes"] == 2 * s["split_blocks"] * 128 * 256 * 4 + s["split_tiles"] * 32
        else:
            assert s["workspace_bytes"] == 0 and s["grid"] == min(s["tiles"], sms)


def test_gemv_schedule_invariants_over_many_shapes(lib):
    """For any shape and SM count: shared memory within the per-block limit, at least two
    ring stages, row blocks that cover N exactly, sweeps that cover M, and a workspace
    exactly when rows are split along K."""
    rng = __import__("random").Random(11)
    for _ in range(400):
        M = rng.choice([1, 2, 3, 4, 5, 8, 16])
        N = rng.choice([1, 8, 100, 1024, 1536, 4096, 14336, 100000])
        K = rng.choice([32, 96, 128, 576, 2880, 4096, 14336, 28672, 65536, 131072])
        g = rng.choice([g for g in (32, 64, 128, 256) if K % g == 0])
        sms = rng.choice([1, 16, 132, 148])
        s = w4.w4a16_gemv_schedule(M, N, K, g, sms)
        assert s["rows_per_sweep"] in (1, 2, 4) and s["rows_per_sweep"] <= max(M, 4)
        assert s["sweeps"] == -(-M // s["rows_per_sweep"])
        assert (s["row_blocks"] - 1) * s["rows_per_block"] < N <= s["row_blocks"] * s["rows_per_block"]
        assert s["smem_bytes"] <= 227 * 1024 and 2 <= s["stages"] <= 16
        assert (s["workspace_bytes"] > 0) == (s["k_parts"] > 1)
        kc = 128 // s["rows_per_sweep"]
        slices = -(-K // kc)
        assert s["k_parts"] >= -(-slices // 448)            # one thread per slice of a part
        assert s["k_parts"] == 1 or s["rows_per_sweep"] == 1  # several activation rows only for whole rows


def test_nf4_levels_of_the_library_equal_the_oracle(lib):
    """The library computes the NF4 levels on the host with its own normal-quantile routine;
    they must equal the oracle's bit for bit (both round the same double values to fp32)."""
    import oracle
    assert np.array_equal(np.array(w4.w4_nf4_levels(), np.float32), oracle.nf4_levels())


def test_gemv_grouped_schedule_fits_one_wave_and_validates(lib):
    """The decode sweep's four GEMVs as one grouped launch: one block per SM at most, each
    problem a share in proportion to its bytes; invalid groups are rejected before any launch."""
    Ks, Ns = [4096, 4096, 4096, 14336], [4096, 1024, 14336, 4096]
    for sms in (148, 132):
        b = w4.w4a16_gemv_grouped_schedule(1, Ns, Ks, 128, sms)
        assert sum(b) <= sms and min(b) >= 1
        assert b[2] > b[0] > b[1]  # more bytes, more blocks
    small = w4.w4a16_gemv_grouped_schedule(1, [77, 5], [320, 4096], 64, 148)
    assert small == [77, 5]  # tiny problems: one row per block within the share
    P = ctypes.c_void_p * 2
    L = ctypes.c_int64 * 2
    ptrs = P(FAKE, FAKE)
    assert rc("w4a16_gemv_grouped", 0, ptrs, 1, ptrs, L(16, 16), L(128, 128), 128, 1, ptrs, 0, None) == 2
    assert rc("w4a16_gemv_grouped", 9, ptrs, 1, ptrs, L(16, 16), L(128, 128), 128, 1, ptrs, 0, None) == 2
    assert rc("w4a16_gemv_grouped", 2, None, 1, ptrs, L(16, 16), L(128, 128), 128, 1, ptrs, 0, None) == 1
    assert rc("w4a16_gemv_grouped", 2, P(FAKE, None), 1, ptrs, L(16, 16), L(128, 128), 128, 1, ptrs, 0, None) == 1
    assert rc("w4a16_gemv_grouped", 2, ptrs, 1, ptrs, L(16, 16), L(128, 96), 64, 1, ptrs, 0, None) == 3
    assert rc("w4a16_gemv_grouped", 2, P(FAKE, FAKE + 8), 1, ptrs, L(16, 16), L(128, 128), 128, 1, ptrs, 0,
              None) == 4
    assert rc("w4a16_gemv_grouped", 2, ptrs, 1, ptrs, L(16, 16), L(128, 128), 128, 3, ptrs, 0, None) == 5
    # rows too long for one block (a K split would need a workspace): unsupported in a group
    assert rc("w4a16_gemv_grouped", 2, ptrs, 1, ptrs, L(16, 16), L(128, 65536), 128, 1, ptrs, 0, None) == 6


@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)])
def test_tc_schedule_of_the_decode_shapes(lib, K, N):
    """The tensor-core W4A16 splits tiles x k-blocks evenly over at most one CTA per SM and
    eight per 128-row tile."""
    s = w4.w4a16_gemm_tc_schedule(4, N, K, 128, 148)
    assert s["tiles"] == N // 128 and s["k_blocks"] == K // 128 and s["k_per_block"] == 128
    # at most 8 CTAs per tile, at most one per SM
    assert s["units"] == s["tiles"] * s["k_blocks"] and s["ctas"] == min(148, 8 * s["tiles"])
    assert s["record_bytes"] == 128 * 64 + 512
    small = w4.w4a16_gemm_tc_schedule(1, 77, 320, 32, 148)
    assert small == {"tiles": 1, "k_blocks": 3, "units": 3, "ctas": 3, "k_per_block": 128,
                     "record_bytes": 128 * 64 + 4 * 512}
    assert rc("w4a16_gemm_tc_schedule", 17, 64, 128, 128, 148, FAKE) == 2
    assert rc("w4a16_gemm_tc_schedule", 1, 64, 128, 96, 148, FAKE) == 3
    assert rc("w4a16_gemm_tc_schedule", 1, 64, 128, 128, 148, None) == 1
