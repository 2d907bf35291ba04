"""Study of the pages' design axis: group size and clip grid.

TAHOMA "MSE clipping" searches 11 contracted ranges (ratios 1.00 ... 0.50) per block; the
decode sweep workload uses 20 ratios over [0.7, 1.0]. QLWG "Granularity" tabulates
weight and output error against group size. This test computes that table with the oracle
on three synthetic layers:
- the single layer with outlier input columns, in the pages' orientation W[576, 1536];
- an 8B-shaped decode layer with 0.1% outlier columns;
- a Student-t(3) layer.
For g in {32, 64, 128, 256}, the GPU quantizer gives the same codes, scales and zero points
bit for bit (tests/test_gpu_quantize.py), and tests/test_gpu_study.py recomputes the output
errors with the GPU quantizer and GEMV. TAHOMA "What the WMT26 paper finds" weighs block 256
against 128 (smaller, faster, worse), which is why 256 is in the table.

Asserted is only what the method guarantees or what these layers show by a wide margin:
- a grid that starts with 1.0 never raises a block's error, so the layer's weight error with
  a clip search is at most its error without one (up to the fp32 rounding of the block
  errors the search compares);
- smaller groups give lower error;
- asymmetric beats symmetric at equal group size.
Run with -s to print the table."""
import numpy as np
import pytest

import oracle
from bit_gemm_wise_b200 import synth

GRIDS = {"none": [1.0], "page 11": synth.clip_grid_page(), "20 in [0.7,1]": synth.clip_grid_20()}
GROUPS = (32, 64, 128, 256)


def layers():
    W, x = synth.single_layer_page_orientation()  # the pages' own table is on W[576, 1536]
    yield "single layer 576x1536, 4 input cols x50", W, synth.normal((16, 1536), 1.0, 0, 900)
    yield "decode 4096x4096 (1024 rows), 0.1% cols x30", synth.decode_weight(4096, 4096)[:1024], \
        synth.decode_activation(16, 4096)
    yield "Student-t(3) q-proj (1024 rows)", synth.llama8b_weight(0, "q")[:1024], synth.normal((16, 4096), 1.0, 0, 901)


def bits_per_weight(mode, g):
    # 16-bit scale per group; the asymmetric zero term is 16-bit as well (TAHOMA "Achievement 1")
    return oracle.bits_per_weight(4, True, g) if mode == "sym" else oracle.bits_per_weight_16bit_zero(4, g)


@pytest.fixture(scope="module")
def table():
    rows = []
    for name, W, X in layers():
        bits = synth.bf16_bits(W)
        w = W.float().numpy().astype(np.float64)
        x = X.float().numpy().astype(np.float64)
        y = x @ w.T
        for mode in ("sym", "asym"):
            for g in GROUPS:
                for gname, grid in GRIDS.items():
                    codes, scales, zeros, _ = oracle.quantize(bits, g, mode, grid, want_chosen=False)
                    wd = oracle.dequantize(codes, scales, zeros, g, mode)
                    rows.append(dict(layer=name, mode=mode, g=g, grid=gname, bpw=bits_per_weight(mode, g),
                                     werr=oracle.rel_error(w, wd), oerr=oracle.rel_error(y, x @ wd.T)))
    print()
    print(f"{'layer':46s} {'mode':5s} {'g':>4s} {'grid':14s} {'bits/w':>6s} {'weight err':>10s} {'output err':>10s}")
    for r in rows:
        print(f"{r['layer']:46s} {r['mode']:5s} {r['g']:4d} {r['grid']:14s} {r['bpw']:6.3f} "
              f"{100 * r['werr']:9.3f}% {100 * r['oerr']:9.3f}%")
    return rows


def pick(rows, **kw):
    out = [r for r in rows if all(r[k] == v for k, v in kw.items())]
    assert len(out) == 1, kw
    return out[0]


def test_clip_search_never_raises_weight_error(table):
    for r in table:
        if r["grid"] == "none":
            continue
        base = pick(table, layer=r["layer"], mode=r["mode"], g=r["g"], grid="none")
        assert r["werr"] <= base["werr"] * (1 + 1e-6), (r, base)


def test_smaller_groups_and_asymmetric_codes_lower_the_error(table):
    for name in {r["layer"] for r in table}:
        for gname in GRIDS:
            for mode in ("sym", "asym"):
                e = [pick(table, layer=name, mode=mode, g=g, grid=gname)["werr"] for g in GROUPS]
                assert all(a < b for a, b in zip(e, e[1:])), (name, mode, gname, e)
            for g in GROUPS:
                assert pick(table, layer=name, mode="asym", g=g, grid=gname)["werr"] < \
                    pick(table, layer=name, mode="sym", g=g, grid=gname)["werr"]
