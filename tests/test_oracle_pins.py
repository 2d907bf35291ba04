"""Pins of the CPU oracle to facts fixed outside it: values the pages print, closed forms,
library routines (numpy float16, torch float8_e4m3fn, numpy fp64 matmul), invariants the
pages state, and brute force. Runs without a GPU."""
import math

import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth
from conftest import load_golden

GOLD = load_golden()


def bf16_bits_of(values):
    t = torch.tensor(np.asarray(values, np.float32)).to(torch.bfloat16)
    return synth.bf16_bits(t)


def golden(key):
    v, tol, _ = GOLD[key]
    return v, tol


# ------------------------------------------------------------------ number formats

def test_fp16_codec_matches_numpy_float16():
    rng = np.random.default_rng(1)
    specials = np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e9, -1e9, 6.0e-8, 2.98e-8,
                         2.9802322e-8, 5.9604645e-8, 6.1035156e-5, 6.1e-5, 1e-30,
                         0.1, 0.08001302, 1.0 / 7.0, 2048.0 + 1.0, 2049.0, 2051.0], np.float32)
    mags = np.exp(rng.uniform(np.log(1e-9), np.log(7e4), 40000)).astype(np.float32)
    vals = np.concatenate([specials, mags, -mags])
    ours = oracle.f32_to_f16_bits(vals)
    ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    # decoding every finite pattern
    pats = np.arange(0, 0x7C00, dtype=np.uint16)
    pats = np.concatenate([pats, pats | 0x8000])
    assert np.array_equal(oracle.f16_bits_to_f32(pats), pats.view(np.float16).astype(np.float32))


def test_fp16_max_is_page_value():
    v, _ = golden("fp16_max")
    assert oracle.f16_bits_to_f32(np.array([0x7BFF], np.uint16))[0] == v
    assert oracle.f32_to_f16_bits(np.array([v], np.float32))[0] == 0x7BFF


def test_e4m3_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    ours = oracle.e4m3_decode(codes)
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    assert np.array_equal(ours[finite], ref[finite])
    v, _ = golden("e4m3_max")
    assert np.nanmax(ours) == v


def test_e4m3_encode_matches_torch_over_all_bf16_times_scales():
    # every finite bf16 pattern, times a few row-scale-like factors, clamped to the finite
    # range (torch's cast does not saturate; ours saturates by definition)
    pats = np.arange(65536, dtype=np.uint32)
    v = (pats << 16).view(np.float32)
    v = v[np.isfinite(v)]
    for scale in (1.0, 448.0 / 3.7, 1.0 / 0.02173):
        x = (v * np.float32(scale)).astype(np.float32)
        x = x[np.isfinite(x)]
        x = np.clip(x, -448.0, 448.0).astype(np.float32)
        ours = oracle.e4m3_encode(x)
        ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(ours, ref), scale


def test_e4m3_encode_saturates():
    x = np.array([448.0, 463.9, 464.0, 500.0, 1e6, -1e6, -470.0], np.float32)
    got = oracle.e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]


# ------------------------------------------------------------------ page numbers

def test_bits_per_weight_table():
    shape = (576, 1536)
    cases = {
        "bpw_int8_sym_per_tensor_576x1536": oracle.bits_per_weight(8, True, shape[0] * shape[1]),
        "bpw_int8_sym_per_channel_576x1536": oracle.bits_per_weight(8, True, shape[1]),
        "bpw_int4_sym_per_tensor_576x1536": oracle.bits_per_weight(4, True, shape[0] * shape[1]),
        "bpw_int4_asym_per_tensor_576x1536": oracle.bits_per_weight(4, False, shape[0] * shape[1]),
        "bpw_int4_sym_per_channel_576x1536": oracle.bits_per_weight(4, True, shape[1]),
        "bpw_int4_asym_per_channel_576x1536": oracle.bits_per_weight(4, False, shape[1]),
        "bpw_int4_sym_g128": oracle.bits_per_weight(4, True, 128),
        "bpw_int4_asym_g128": oracle.bits_per_weight(4, False, 128),
        "bpw_int4_sym_g32": oracle.bits_per_weight(4, True, 32),
        "bpw_int4_asym_g32": oracle.bits_per_weight(4, False, 32),
        "bpw_int3_asym_g128": oracle.bits_per_weight(3, False, 128),
        "bpw_int3_asym_g32": oracle.bits_per_weight(3, False, 32),
        "bpw_tahoma_g128_16bit_zero": oracle.bits_per_weight_16bit_zero(4, 128),
    }
    for key, got in cases.items():
        v, tol = golden(key)
        assert abs(got - v) <= tol + 1e-12, (key, got, v)
    v, _ = golden("bpw_fp16_scale_g128_overhead")
    assert oracle.bits_per_weight(4, True, 128) - 4 == v


def test_int4_per_tensor_step_of_page_layer():
    # a tensor whose max |w| is the page's 5.812: per-tensor symmetric INT4 step 5.8/7 = 0.83
    rng = np.random.default_rng(0)
    w = rng.normal(0, 0.2, size=(576, 1536))
    w[3, 5] = 5.812
    _, scales = oracle.fake_quant(w, 4, True, None)
    v, tol = golden("int4_per_tensor_step_max_5.812")
    assert abs(scales[0] - v) <= tol
    # "almost everything rounds to zero"
    wq, _ = oracle.fake_quant(w, 4, True, None)
    assert np.mean(wq == 0) > 0.9


def test_int8_outlier_example():
    # one 8.5 among values of magnitude ~0.01, INT8 per-tensor symmetric
    rng = np.random.default_rng(2)
    x = rng.choice([-1.0, 1.0], 4096) * rng.uniform(0.005, 0.015, 4096)
    x[1234] = 8.5
    xq, scales = oracle.fake_quant(x, 8, True, None)
    v, tol = golden("int8_outlier_scale_8.5")
    assert abs(scales[0] - v) <= tol
    assert scales[0] == 8.5 / 127
    small = np.ones(x.size, bool)
    small[1234] = False
    # the small values collapse onto a few integer levels near zero (codes -0, 0 only here)
    codes = np.rint(x[small] / scales[0])
    assert set(np.unique(codes)) <= {-1.0, 0.0, 1.0}
    assert np.mean(codes == 0) > 0.9
    # the per-value error bound scale/2
    assert np.max(np.abs(x - xq)) <= scales[0] / 2 + 1e-15


def test_block_example_steps_and_zero_point():
    # [-0.2, 1.0]: symmetric step ~ 1/7 = 0.143, affine step 1.2/15 = 0.08 (before rounding)
    blk = np.linspace(-0.2, 1.0, 128)
    _, s_sym = oracle.fake_quant(blk, 4, True, 128)
    _, s_asym = oracle.fake_quant(blk, 4, False, 128)
    v, tol = golden("sym_step_block_-0.2_1.0")
    assert abs(s_sym[0] - v) <= tol
    v, tol = golden("asym_step_block_-0.2_1.0")
    assert abs(s_asym[0] - v) <= tol
    # the same block through the INT4 oracle (bf16 input, fp16 scale storage)
    bits = bf16_bits_of(blk)
    for mode, step_key in (("sym", "sym_step_block_-0.2_1.0"), ("asym", "asym_step_block_-0.2_1.0")):
        codes, scales, zeros, _ = oracle.quantize(bits[None, :], 128, mode, [1.0])
        s = oracle.f16_bits_to_f32(scales)[0, 0]
        v, _ = golden(step_key)
        assert abs(s - v) < 2e-3
    # asymmetric uses all 16 codes on this block, symmetric at most 15 and never code -8
    codes, _, _, _ = oracle.quantize(bits[None, :], 128, "asym", [1.0])
    v, _ = golden("int4_asym_levels_used")
    assert len(np.unique(oracle.unpack_codes(codes))) == v
    codes, _, _, _ = oracle.quantize(bits[None, :], 128, "sym", [1.0])
    used = np.unique(oracle.unpack_codes(codes))
    v, _ = golden("int4_sym_levels_used")
    assert len(used) <= v and 0 not in used


def test_zero_point_rounds_half_to_even():
    # lo = -0.3125, hi = 1.5625: s = 1.875/15 = 0.125 exactly, -lo/s = 2.5 exactly
    blk = np.full(32, 0.5, np.float32)
    blk[0], blk[1] = -0.3125, 1.5625
    codes, scales, zeros, _ = oracle.quantize(bf16_bits_of(blk)[None, :], 32, "asym", [1.0])
    assert oracle.f16_bits_to_f32(scales)[0, 0] == 0.125
    assert zeros[0, 0] == 2           # half-to-even (round-half-up would give 3)
    # a code tie: w/s = 4.5 -> 4, 5.5 -> 6
    blk2 = blk.copy()
    blk2[2], blk2[3] = 4.5 * 0.125, 5.5 * 0.125
    codes, _, zeros, _ = oracle.quantize(bf16_bits_of(blk2)[None, :], 32, "asym", [1.0])
    q = oracle.unpack_codes(codes)[0]
    assert q[2] == 4 + 2 and q[3] == 6 + 2


def test_zero_range_guard():
    z = np.zeros((2, 64), np.float32)
    for mode in ("sym", "asym"):
        codes, scales, zeros, _ = oracle.quantize(bf16_bits_of(z), 64, mode, synth.clip_grid_20())
        assert np.all(scales == 0x3C00)           # fp16 1.0
        W = oracle.dequantize(codes, scales, zeros, 64, mode)
        assert np.all(W == 0)


# ------------------------------------------------------------------ quantizer invariants

def _rand_weights(N, K, seed, outliers=0):
    w = synth.outlier_weight(N, K, outliers, 30.0, seed, 7)
    return synth.bf16_bits(w), w.float().numpy().astype(np.float64)


@pytest.mark.parametrize("g", [32, 64, 128, 256])
def test_sym_never_emits_minus8_and_error_bound(g):
    bits, w = _rand_weights(64, 1024, 3, outliers=3)
    codes, scales, _, _ = oracle.quantize(bits, g, "sym", [1.0])
    q = oracle.unpack_codes(codes)
    assert q.min() >= 1          # nibble 0 is code -8
    assert q.max() <= 15
    W = oracle.dequantize(codes, scales, None, g, "sym")
    s = np.repeat(oracle.f16_bits_to_f32(scales).astype(np.float64), g, axis=1)
    # |w - w'| <= s/2, up to the fp16 rounding of the scale (7 * 2^-11 steps at the ends)
    assert np.all(np.abs(w - W) <= s * (0.5 + 7 * 2.0 ** -11) + 1e-12)


@pytest.mark.parametrize("g", [32, 128])
def test_asym_error_bound_at_full_range(g):
    bits, w = _rand_weights(64, 1024, 4, outliers=3)
    codes, scales, zeros, _ = oracle.quantize(bits, g, "asym", [1.0])
    W = oracle.dequantize(codes, scales, zeros, g, "asym")
    s = np.repeat(oracle.f16_bits_to_f32(scales).astype(np.float64), g, axis=1)
    assert np.all(np.abs(w - W) <= s * (0.5 + 15 * 2.0 ** -11) + 1e-12)
    # plain min/max: every group's extremes are inside the reconstruction lattice range
    q = oracle.unpack_codes(codes)
    assert q.min() == 0 and q.max() == 15


def test_grid_one_matches_page_fake_quant_up_to_fp16_scale():
    """With the single ratio 1.0 the INT4 oracle is the plain group quantizer of the
    'Quantize, then dequantize' fake_quant; the only difference is the fp16 scale storage,
    so the reconstructions agree to within one step of the fp16 rounding."""
    bits, w = _rand_weights(32, 576, 5, outliers=2)
    for mode, sym in (("sym", True), ("asym", False)):
        codes, scales, zeros, _ = oracle.quantize(bits, 32, mode, [1.0])
        W = oracle.dequantize(codes, scales, zeros, 32, mode)
        ref, s_ref = oracle.fake_quant(w, 4, sym, 32)
        s = np.repeat(s_ref.reshape(32, -1), 32, axis=1)
        diff = np.abs(W - ref)
        # identical codes except where the fp16 scale moves a value across a rounding edge
        assert np.mean(diff <= 16 * 2.0 ** -11 * s + 1e-12) > 0.99
        assert np.all(diff <= s * 1.01 + 1e-12)


def test_outlier_isolation_under_group_quant():
    """One weight set to 10x the tensor max: under group quantization every other group keeps
    exactly its codes and scale; under per-tensor INT8 the other rows' error grows."""
    bits, w = _rand_weights(16, 512, 6)
    ws = w.copy()
    ws[7, 100] = 10 * np.abs(w).max()
    bits_s = bf16_bits_of(ws)
    a = oracle.quantize(bits, 128, "asym", synth.clip_grid_20())
    b = oracle.quantize(bits_s, 128, "asym", synth.clip_grid_20())
    touched = np.zeros((16, 4), bool)
    touched[7, 0] = True
    for x, y in zip(a[1:], b[1:]):
        assert np.array_equal(x[~touched], y[~touched])
    ca, cb = a[0].reshape(16, 4, 64), b[0].reshape(16, 4, 64)
    assert np.array_equal(ca[~touched], cb[~touched])
    # per-tensor INT8 on the same matrices: rows other than 7 get much worse
    others = np.ones(16, bool)
    others[7] = False
    wq, _ = oracle.fake_quant(w, 8, True, None)
    wsq, _ = oracle.fake_quant(ws, 8, True, None)
    e0 = oracle.rel_error(w[others], wq[others])
    e1 = oracle.rel_error(ws[others], wsq[others])
    assert e1 > 5 * e0
    # per-channel leaves them exactly where they were
    wq, _ = oracle.fake_quant(w, 8, True, 512)
    wsq, _ = oracle.fake_quant(ws, 8, True, 512)
    assert oracle.rel_error(w[others], wq[others]) == oracle.rel_error(ws[others], wsq[others])


def test_group_error_ordering_trends():
    """Weak trend checks of the page's table on synthetic data: asym < sym, g32 < g128 <
    per-channel."""
    bits, w = _rand_weights(128, 1536, 8, outliers=2)
    err = {}
    for mode in ("sym", "asym"):
        for g in (32, 128):
            codes, scales, zeros, _ = oracle.quantize(bits, g, mode, [1.0])
            err[(mode, g)] = oracle.rel_error(w, oracle.dequantize(codes, scales, zeros, g, mode))
    pc, _ = oracle.fake_quant(w, 4, True, 1536)
    assert err[("asym", 128)] < err[("sym", 128)]
    assert err[("asym", 32)] < err[("sym", 32)]
    assert err[("sym", 32)] < err[("sym", 128)] < oracle.rel_error(w, pc)


# ------------------------------------------------------------------ clip search

def _candidate_fp64(w32, mode, r):
    """Independent brute force of one candidate: numpy fp32 for the scale/zero/code steps
    (the precision the pages' method decides codes in), fp64 for the block error."""
    f32 = np.float32
    if mode == "sym":
        a = np.max(np.abs(w32))
        s = np.float16(f32(r) * a / f32(7.0)).astype(f32)
        if s == 0:
            s = f32(1.0)
        c = np.clip(np.rint(w32 / s), -7, 7)
        rec = (c * s).astype(f32)
    else:
        lo, hi = w32.min(), w32.max()
        h = f32(0.5) * (hi - lo)
        cc = (f32(1.0) - f32(r)) * h
        lo_r, hi_r = lo + cc, hi - cc
        s = np.float16((hi_r - lo_r) / f32(15.0)).astype(f32)
        if s == 0:
            s = f32(1.0)
        z = np.clip(np.rint(-lo_r / s), -32768, 32767)
        q = np.clip(np.rint(w32 / s) + z, 0, 15)
        rec = ((q - z).astype(f32) * s).astype(f32)
    return float(np.sum((w32.astype(np.float64) - rec.astype(np.float64)) ** 2))


@pytest.mark.parametrize("mode", ["sym", "asym"])
@pytest.mark.parametrize("g", [32, 128, 256])
def test_clip_search_is_brute_force_argmin(mode, g):
    rng = np.random.default_rng(11)
    grid = synth.clip_grid_20()
    N = 48
    w = rng.standard_t(3, size=(N, g)).astype(np.float32) * 0.02
    w[::5, 3] *= 40.0                  # some blocks with one far outlier
    bits = bf16_bits_of(w)
    w32 = oracle.bf16_to_f32(bits)
    codes, scales, zeros, chosen = oracle.quantize(bits, g, mode, grid)
    n_outlier_clipped = 0
    for n in range(N):
        sse = np.array([_candidate_fp64(w32[n], mode, r) for r in grid])
        i = int(chosen[n, 0])
        best = sse.min()
        # the chosen ratio is optimal, up to near-ties decided by fp32 rounding
        assert sse[i] <= best * (1 + 1e-5) + 1e-30, (n, i, sse[i], best)
        # never worse than the full range
        assert sse[i] <= sse[0] * (1 + 1e-6) + 1e-30
        # the oracle's own candidate errors: chosen is the first strict minimum
        own = np.array([oracle.block_sse(bits[n], mode, r) for r in grid], np.float32)
        first = 0
        for k in range(1, len(grid)):
            if own[k] < own[first]:
                first = k
        assert i == first
        if n % 5 == 0 and i > 0:
            n_outlier_clipped += 1
    # blocks with one far outlier usually contract the range
    assert n_outlier_clipped >= 3


def test_clip_search_grid_one_equals_plain():
    bits, _ = _rand_weights(16, 256, 9)
    a = oracle.quantize(bits, 128, "asym", [1.0])
    b = oracle.quantize(bits, 128, "asym", [1.0, 1.0, 1.0])
    for x, y in zip(a[:3], b[:3]):
        assert np.array_equal(x, y)
    assert np.all(b[3] == 0)


def test_page_grid_shape():
    g = synth.clip_grid_page()
    v, _ = golden("page_clip_ratio_count")
    assert len(g) == v and g[0] == 1.0 and abs(g[-1] - 0.5) < 1e-7
    g20 = synth.clip_grid_20()
    assert len(g20) == 20 and g20[0] == 1.0 and abs(g20[-1] - 0.7) < 1e-7


# ------------------------------------------------------------------ activations

def test_row_quant_invariants():
    X = synth.outlier_activation(64, 512, 8, 20.0, 0, 3)
    X = X.clone()
    X[5] = 0
    bits = synth.bf16_bits(X)
    X8, s, G = oracle.row_quant(bits, 128)
    x = X.float().numpy()
    # all-zero row stays zero, 1e-8 floor
    assert np.all(X8[5] == 0)
    assert s[5] == np.float32(np.float32(1e-8) / np.float32(448.0))
    # every non-zero row reaches +-448
    for m in range(64):
        if m != 5:
            assert np.any((X8[m] & 0x7F) == 0x7E)
    # scale = rowmax/448
    amax = np.abs(x).max(axis=1)
    ref_s = (np.maximum(amax, np.float32(1e-8)) / np.float32(448.0)).astype(np.float32)
    assert np.array_equal(s, ref_s)
    # codes are torch's E4M3 cast of x/s
    ref = torch.from_numpy((x / s[:, None]).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(X8, ref)
    # dequantized error: at most half an E4M3 step (relative 2^-4 normal, 2^-10 * s subnormal)
    deq = oracle.e4m3_decode(X8).astype(np.float64) * s[:, None]
    err = np.abs(deq - x)
    assert np.all(err <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * s[:, None]) + 1e-30)
    # group sums: exact fp64 sum of the decoded values, rounded once to fp32
    ref_G = oracle.e4m3_decode(X8).astype(np.float64).reshape(64, 4, 128).sum(-1).astype(np.float32)
    assert np.array_equal(G, ref_G)


# ------------------------------------------------------------------ reference products

def test_gemv_ref_matches_numpy_matmul_and_closed_forms():
    bits, _ = _rand_weights(96, 512, 10, outliers=1)
    codes, scales, zeros, _ = oracle.quantize(bits, 128, "asym", synth.clip_grid_20())
    x = synth.normal((4, 512), 1.0, 0, 99)
    xb = synth.bf16_bits(x)
    y = oracle.gemv_ref(xb, codes, scales, zeros, 128, "asym")
    Wd = oracle.dequantize(codes, scales, zeros, 128, "asym")
    ref = x.double().numpy() @ Wd.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    # one-hot x picks a column of the dequantized weight
    oh = np.zeros((1, 512), np.float32)
    oh[0, 77] = 1.0
    y1 = oracle.gemv_ref(bf16_bits_of(oh), codes, scales, zeros, 128, "asym")
    assert np.array_equal(y1[0], Wd[:, 77])
    # q == z everywhere -> y == 0
    z8 = np.full_like(zeros, 8)
    c8 = np.full_like(codes, 0x88)
    assert np.all(oracle.gemv_ref(xb, c8, scales, z8, 128, "asym") == 0)


def test_dequantize_closed_form():
    codes = np.array([[0x10, 0xF8]], np.uint8)     # q = 0, 1, 8, 15
    scales = oracle.f32_to_f16_bits(np.array([[0.5]], np.float32))
    zeros = np.array([[3]], np.int16)
    W = oracle.dequantize(np.pad(codes, ((0, 0), (0, 14))), scales, zeros, 32, "asym")
    assert list(W[0, :4]) == [-1.5, -1.0, 2.5, 6.0]
    Ws = oracle.dequantize(np.pad(codes, ((0, 0), (0, 14))), scales, None, 32, "sym")
    assert list(Ws[0, :4]) == [-4.0, -3.5, 0.0, 3.5]


def test_w4a8_ref_pairs_matches_dense():
    bits, _ = _rand_weights(64, 256, 12)
    codes, scales, zeros, _ = oracle.quantize(bits, 32, "asym", [1.0])
    X = synth.outlier_activation(16, 256, 2, 20.0, 0, 5)
    X8, s, _ = oracle.row_quant(synth.bf16_bits(X), 32)
    dense = oracle.w4a8_ref_dense(X8, s, codes, scales, zeros, 32, "asym")
    rows, cols = np.meshgrid(np.arange(16), np.arange(64), indexing="ij")
    pairs = oracle.w4a8_ref_pairs(X8, s, codes, scales, zeros, 32, "asym", rows.ravel(), cols.ravel())
    assert np.allclose(pairs.reshape(16, 64), dense, rtol=1e-12, atol=1e-12)
    # closed form: the W4A8 operands are the dequantized ones; against the bf16 input the
    # product differs only by the E4M3 rounding of the activations (relative <= 2^-4)
    Wd = oracle.dequantize(codes, scales, zeros, 32, "asym")
    exact = X.double().numpy() @ Wd.T
    assert oracle.rel_error(exact, dense) < 2.0 ** -4


@pytest.mark.parametrize("mode", ["sym", "asym"])
def test_codes_are_nearest_lattice_points_of_stored_scale(mode):
    """Every code strictly inside the code range is the nearest lattice point of the STORED
    (fp16) scale and zero: |w/s + z - q| <= 1/2 (rounding the fp32 quotient can move a tie
    by one ulp). This is the "error <= scale/2" bound of the pages applied to the stored
    representation, and it fails if codes are taken from the unrounded scale."""
    bits, w = _rand_weights(128, 1024, 13, outliers=3)
    g = 128
    codes, scales, zeros, _ = oracle.quantize(bits, g, mode, synth.clip_grid_20())
    q = oracle.unpack_codes(codes).astype(np.float64)
    s = np.repeat(oracle.f16_bits_to_f32(scales).astype(np.float64), g, axis=1)
    z = 8.0 if mode == "sym" else np.repeat(zeros.astype(np.float64), g, axis=1)
    inner = (q > (1 if mode == "sym" else 0)) & (q < 15)
    d = np.abs(w / s + z - q)
    assert np.all(d[inner] <= 0.5 + 1e-5)


def test_block_sse_closed_form():
    # lattice values k * 0.125 (s = 0.875 / 7 = 0.125 exactly in fp16) plus one value off the
    # lattice by 1/32: the block error is exactly (1/32)^2
    blk = (np.arange(32) % 15 - 7).astype(np.float32) * np.float32(0.125)
    blk[4] = np.float32(3 * 0.125 + 0.03125)
    sse = oracle.block_sse(bf16_bits_of(blk), "sym", 1.0)
    assert sse == 2.0 ** -10


def test_row_quant_floor_below_1e8():
    X = np.zeros((2, 64), np.float32)
    X[0, :] = 3e-9
    X[1, :] = -5e-7
    X8, s, _ = oracle.row_quant(bf16_bits_of(X), 0)
    # amax below the floor: the scale is the floor / 448 and codes stay small
    assert s[0] == np.float32(np.float32(1e-8) / np.float32(448.0))
    assert np.all((X8[0] & 0x7F) < 0x7E)
    # amax above the floor: the scale is amax / 448
    a = np.float32(oracle.bf16_to_f32(bf16_bits_of(X[1:2]))[0, 0])
    assert s[1] == np.float32(np.abs(a) / np.float32(448.0))


# ------------------------------------------------------------------ mixture-of-experts layer

def test_moe_route_topk_and_softmax_gates():
    """Top-k against numpy's stable argsort of the negated logits (ties to the lower expert),
    gates against scipy's softmax of the selected logits; a two-expert closed form."""
    from scipy.special import softmax
    rng = np.random.default_rng(21)
    lg = rng.random((300, 32)).astype(np.float32)
    lg[7, [3, 9, 12]] = lg[7].max() + 0.5      # a three-way tie at the top
    ex, g = oracle.moe_route(lg, 4)
    ref = np.argsort(-lg, axis=1, kind="stable")[:, :4]
    assert np.array_equal(ex, ref)
    assert list(ex[7, :3]) == [3, 9, 12]
    sel = np.take_along_axis(lg.astype(np.float64), ref, axis=1)
    assert np.allclose(g, softmax(sel, axis=1), rtol=1e-14, atol=0)
    assert np.allclose(g.sum(1), 1.0, rtol=0, atol=1e-15)
    # k = 2, logits a > b: gates 1 / (1 + e^(b - a)) and the rest
    ex2, g2 = oracle.moe_route(np.array([[0.0, 2.0, 0.5]], np.float32), 2)
    assert list(ex2[0]) == [1, 2]
    assert abs(g2[0, 0] - 1.0 / (1.0 + np.exp(-1.5))) < 1e-15


def test_moe_grouping_covers_every_pair_once():
    rng = np.random.default_rng(22)
    lg = rng.random((64, 8)).astype(np.float32)
    ex, _ = oracle.moe_route(lg, 3)
    tor, off, row_of = oracle.moe_grouping(ex, 8)
    assert off[0] == 0 and off[-1] == 64 * 3 and np.all(np.diff(off) >= 0)
    seen = set()
    for t in range(64):
        for i in range(3):
            r = row_of[t, i]
            assert tor[r] == t and off[ex[t, i]] <= r < off[ex[t, i] + 1]
            seen.add(int(r))
    assert seen == set(range(64 * 3))
    for e in range(8):  # tokens ascending inside an expert
        assert np.all(np.diff(tor[off[e]:off[e + 1]]) > 0)


def test_swiglu_row_quant_against_library_sigmoid_and_codec():
    """h = gate * sigmoid(gate) * up against scipy's expit in fp64 (rounded to fp32); the
    codes against torch's float8_e4m3fn cast of h / s; closed forms silu(0) = 0 and
    silu(v) - silu(-v) = v."""
    from scipy.special import expit
    rng = np.random.default_rng(23)
    H = 96
    g = rng.normal(0, 3, (5, H)).astype(np.float32)
    u = rng.normal(0, 1, (5, H)).astype(np.float32)
    g[0, :4] = [0.0, -0.0, 40.0, -40.0]
    Y = torch.from_numpy(np.concatenate([g, u], 1)).to(torch.bfloat16)
    gb, ub = Y[:, :H].double().numpy(), Y[:, H:].double().numpy()
    X8, s, h = oracle.swiglu_row_quant(synth.bf16_bits(Y), H)
    ref = (gb * expit(gb) * ub).astype(np.float32)
    assert np.array_equal(h, ref)
    assert h[0, 0] == 0.0 and h[0, 1] == 0.0
    amax = np.abs(h).max(1)
    assert np.array_equal(s, (np.maximum(amax, np.float32(1e-8)) / np.float32(448.0)).astype(np.float32))
    q = (torch.from_numpy(h) / torch.from_numpy(s)[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(X8, q)
    # silu(v) - silu(-v) = v with up = 1
    v = np.linspace(-6, 6, H).astype(np.float32)
    Y2 = torch.from_numpy(np.stack([np.concatenate([v, np.ones(H, np.float32)]),
                                    np.concatenate([-v, np.ones(H, np.float32)])])).to(torch.bfloat16)
    vb = Y2[0, :H].double().numpy()
    _, _, h2 = oracle.swiglu_row_quant(synth.bf16_bits(Y2), H)
    assert np.allclose(h2[0].astype(np.float64) - h2[1], vb, rtol=0, atol=4e-6 * np.abs(vb).max())


def test_moe_combine_against_einsum_and_one_hot():
    rng = np.random.default_rng(24)
    rows = rng.normal(0, 1, (40, 17))
    row_of = rng.permutation(40).reshape(10, 4).astype(np.int32)
    gates = rng.random((10, 4))
    y = oracle.moe_combine(rows, row_of, gates)
    assert np.allclose(y, np.einsum("tk,tkn->tn", gates, rows[row_of]), rtol=1e-14, atol=1e-14)
    onehot = np.zeros((10, 4))
    onehot[:, 2] = 1.0
    assert np.array_equal(oracle.moe_combine(rows, row_of, onehot), rows[row_of[:, 2]])


def test_moe_layer_ref_matches_independent_numpy_composition():
    """The layer reference against a composition written here from numpy / torch library
    routines only (argsort, softmax, matmul, float8 cast, expit), at a tiny size."""
    from scipy.special import expit, softmax
    E, k, T, K, H, g = 4, 2, 12, 64, 32, 32
    rng = np.random.default_rng(25)
    X = torch.from_numpy(rng.normal(0, 1, (T, K)).astype(np.float32)).to(torch.bfloat16)
    lg = rng.random((T, E)).astype(np.float32)
    gu = [oracle.quantize(synth.bf16_bits(synth.normal((2 * H, K), 0.02, 9, e)), g, "asym", [1.0], False)[:3]
          for e in range(E)]
    dn = [oracle.quantize(synth.bf16_bits(synth.normal((K, H), 0.02, 9, 50 + e)), g, "asym", [1.0], False)[:3]
          for e in range(E)]
    stack = lambda L: tuple(np.stack([x[i] for x in L]) for i in range(3))
    y, _ = oracle.moe_layer_ref(synth.bf16_bits(X), lg, k, stack(gu), stack(dn), g, "asym")

    def e4m3_rows(a):  # per-row E4M3 quantization with torch's codec
        a = torch.from_numpy(np.asarray(a, np.float32))
        s = torch.clamp(a.abs().amax(1), min=1e-8) / 448.0
        return (a / s[:, None]).to(torch.float8_e4m3fn).double() * s.double()[:, None]

    ref = np.zeros((T, K))
    order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
    for t in range(T):
        w = softmax(lg[t, order[t]].astype(np.float64))
        a = e4m3_rows(X[t:t + 1].float().numpy())
        for i, e in enumerate(order[t]):
            Wgu = oracle.dequantize(*gu[e], g, "asym")
            z = torch.from_numpy(a.numpy() @ Wgu.T).float().to(torch.bfloat16).double().numpy()
            hh = (z[:, :H] * expit(z[:, :H]) * z[:, H:]).astype(np.float32)
            o = e4m3_rows(hh).numpy() @ oracle.dequantize(*dn[e], g, "asym").T
            ref[t] += w[i] * o[0]
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ NF4 comparator

def test_nf4_levels_are_normal_quantiles():
    """The levels against scipy's normal quantile function (an independent inverse CDF):
    eight positive and seven negative quantiles at equal probability steps from 1 - delta
    towards 1/2, delta = (1/32 + 1/30) / 2, an exact zero, scaled to [-1, 1]."""
    from scipy.stats import norm
    v = oracle.nf4_levels().astype(np.float64)
    d = 0.5 * (1 / 32 + 1 / 30)
    top = norm.ppf(1 - d)
    pos = norm.ppf(np.linspace(1 - d, 0.5, 9)[:-1]) / top
    neg = -norm.ppf(np.linspace(1 - d, 0.5, 8)[:-1]) / top
    ref = np.sort(np.concatenate([pos, [0.0], neg])).astype(np.float32)
    assert np.allclose(v, ref, rtol=0, atol=2e-7)
    assert v[7] == 0.0 and v[0] == -1.0 and v[15] == 1.0 and np.all(np.diff(v) > 0)
    # equal probability steps: Phi(level * top) on the positive side
    p = norm.cdf(v[8:] * top)
    assert np.allclose(np.diff(p), (1 - d - 0.5) / 8, rtol=0, atol=1e-6)


def test_nf4_quantize_is_nearest_level_per_block():
    rng = np.random.default_rng(31)
    W = torch.from_numpy(rng.normal(0, 0.02, (40, 256)).astype(np.float32))
    W[3, 64:128] = 0.0
    W[5, :64] = torch.linspace(-1, 1, 64)
    Wb = W.to(torch.bfloat16)
    codes, a = oracle.nf4_quantize(synth.bf16_bits(Wb))
    w = Wb.float().numpy()
    lv = oracle.nf4_levels()
    blocks = w.reshape(40, 4, 64)
    amax = np.abs(blocks).max(2)
    assert np.array_equal(a, amax.astype(np.float32))
    t = np.divide(blocks, amax[:, :, None], out=np.zeros_like(blocks), where=amax[:, :, None] > 0).astype(np.float32)
    q = np.argmin(np.abs(t[..., None] - lv).astype(np.float32), axis=-1)
    q[amax == 0] = 7
    q = q.reshape(40, 256)
    assert np.array_equal(oracle.unpack_codes(codes), q)


def test_nf4_gemv_ref_matches_numpy():
    rng = np.random.default_rng(32)
    Wb = torch.from_numpy(rng.normal(0, 0.02, (24, 192)).astype(np.float32)).to(torch.bfloat16)
    codes, a = oracle.nf4_quantize(synth.bf16_bits(Wb))
    x = torch.from_numpy(rng.normal(0, 1, (3, 192)).astype(np.float32)).to(torch.bfloat16)
    Wd = oracle.nf4_levels().astype(np.float64)[oracle.unpack_codes(codes)] * np.repeat(a.astype(np.float64), 64, 1)
    ref = x.double().numpy() @ Wd.T
    assert np.allclose(oracle.nf4_gemv_ref(synth.bf16_bits(x), codes, a), ref, rtol=1e-13, atol=1e-13)
