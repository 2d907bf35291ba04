"""GPU w4a16_gemv vs the CPU oracle's fp64 product of the dequantized weight.

Tolerances (relative Frobenius): bf16 output against the fp64 result rounded to bf16 at
1e-3 (the required bound); fp32 output against the unrounded fp64 result at 1e-4. The
kernel holds each slice of activations as 24-bit fixed point with one exponent per slice
(|X| < 2^19, so every value within 2^11 of the slice's largest is exact and smaller ones are
off by at most 2^-20 of that largest), forms the integer products with the codes exactly,
and rounds in fp32 only when it combines a group segment and adds the row: the expected
error is ~1e-6 relative, so 1e-4 leaves a margin of about 100."""
import functools

import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import bf16_round, cuda, np_of, rel_frob, to_dev

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def quantized(kind, K, N, group, mode, grid_name):
    if kind == "decode":
        W = synth.decode_weight(K, N)
    elif kind == "single":
        W, _ = synth.single_layer()
    else:
        W = synth.student_t3_weight(N, K, 3, 700 + N + K)
    grid = {"one": [1.0], "twenty": synth.clip_grid_20()}[grid_name]
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), group, mode, grid, want_chosen=False)
    return codes, scales, zeros


def gpu_gemv(codes, scales, zeros, N, K, group, mode, x_bits, out_fp32):
    M = x_bits.shape[0]
    packed = w4.alloc_packed(N, K, group, w4.W4_LAYOUT_GEMV)
    c = to_dev(codes)
    s = to_dev(scales.view(np.int16))
    z = to_dev(zeros) if zeros is not None else None
    w4.w4_prepack(c, s, z, N, K, group, mode, w4.W4_LAYOUT_GEMV, packed)
    x = to_dev(x_bits.view(np.int16)).view(torch.bfloat16)
    # NaN-filled, so that an output the kernel does not write cannot pass as a stale value
    y = torch.full((M, N), float("nan"), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=cuda())
    ws = w4.alloc_gemv_workspace(N, K, group)
    w4.w4a16_gemv(x, M, packed, N, K, group, mode, y, out_fp32, ws)
    torch.cuda.synchronize()
    assert w4.w4_device_status() == 0
    out = y.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(out).all(), f"unwritten outputs in rows {np.unique(np.nonzero(~np.isfinite(out))[1])[:20]}"
    return out


def check(codes, scales, zeros, group, mode, x_bits):
    N, K = codes.shape[0], codes.shape[1] * 2
    ref = oracle.gemv_ref(x_bits, codes, scales, zeros, group, mode)
    y32 = gpu_gemv(codes, scales, zeros, N, K, group, mode, x_bits, 1)
    e32 = rel_frob(ref, y32)
    bad = np.nonzero(np.abs(y32 - ref).max(axis=0) > 1e-3 * np.abs(ref).max())[0]
    assert e32 <= 1e-4, (e32, len(bad), bad[:20].tolist())
    y16 = gpu_gemv(codes, scales, zeros, N, K, group, mode, x_bits, 0)
    e16 = rel_frob(bf16_round(ref), y16)
    assert e16 <= 1e-3, e16
    return e32, e16


def test_single_layer_m1():
    codes, scales, zeros = quantized("single", 576, 1536, 32, "sym", "one")
    _, x = synth.single_layer()
    check(codes, scales, None, 32, "sym", synth.bf16_bits(x))


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
@pytest.mark.parametrize("M", synth.DECODE_M)
def test_decode_sweep_full_size(K, N, M):
    codes, scales, zeros = quantized("decode", K, N, 128, "asym", "twenty")
    x = synth.decode_activation(M, K)
    check(codes, scales, zeros, 128, "asym", synth.bf16_bits(x))


@pytest.mark.parametrize("M", [1, 2, 3, 5, 9, 16])
@pytest.mark.parametrize("group,mode", [(32, "sym"), (64, "asym"), (128, "asym"), (128, "sym"), (256, "asym")])
def test_ragged(M, group, mode):
    N = 77                              # not a multiple of 8
    K = 320 if group < 128 else (384 if group == 128 else 768)  # 320, 384: not multiples of 256
    codes, scales, zeros = quantized("t3", K, N, group, mode, "twenty")
    x = synth.normal((M, K), 1.0, 4, 31 * M + group)
    check(codes, scales, zeros, group, mode, synth.bf16_bits(x))


def test_tiny():
    for N, K, g in [(1, 32, 32), (8, 128, 128), (9, 64, 32)]:
        codes, scales, zeros = quantized("t3", K, N, g, "asym", "one")
        x = synth.normal((1, K), 1.0, 5, N + K)
        check(codes, scales, zeros, g, "asym", synth.bf16_bits(x))


def test_extreme_zero_points():
    """Blocks far from zero make |z| large (one-signed blocks); the chunk offset removal
    must still be exact to fp32 rounding."""
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (64, 256))
    blocks = W.reshape(64, 8, 32)
    pick = rng.integers(0, 3, (64, 8))
    blocks[pick == 1] = 1.0 + rng.uniform(0, 0.02, (int((pick == 1).sum()), 32))     # z far below 0
    blocks[pick == 2] = -3.0 - rng.uniform(0, 0.05, (int((pick == 2).sum()), 32))    # z far above 15
    W = blocks.reshape(64, 256)
    bits = synth.bf16_bits(torch.tensor(W, dtype=torch.float32).to(torch.bfloat16))
    codes, scales, zeros, _ = oracle.quantize(bits, 32, "asym", synth.clip_grid_20(), want_chosen=False)
    assert np.abs(zeros).max() > 241
    x = synth.normal((4, 256), 1.0, 6, 1)
    check(codes, scales, zeros, 32, "asym", synth.bf16_bits(x))


def test_one_hot_column():
    codes, scales, zeros = quantized("t3", 256, 64, 128, "asym", "one")
    x = np.zeros((1, 256), np.float32)
    x[0, 131] = 1.0
    xb = synth.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    y = gpu_gemv(codes, scales, zeros, 64, 256, 128, "asym", xb, 1)
    Wd = oracle.dequantize(codes, scales, zeros, 128, "asym")
    assert np.array_equal(y[0], Wd[:, 131])


@pytest.mark.parametrize("regime", ["tiny", "subnormal_mix", "huge", "zero_slices", "wide_slice"])
def test_activations_far_from_one(regime):
    """The per-slice exponent must follow the activations over the bf16 range: tiny values
    (with bf16 subnormals among them), huge values, all-zero slices, and a slice whose values
    span more than 2^11 (the small ones are then rounded to 2^-20 of the largest)."""
    K, N = 1024, 40
    codes, scales, zeros = quantized("t3", K, N, 128, "asym", "one")
    x = synth.normal((1, K), 1.0, 8, 3).float()
    if regime == "tiny":
        x *= 1e-35
    elif regime == "subnormal_mix":
        x *= 1e-36
        x[0, ::7] *= 1e-3          # bf16 subnormals next to normal values of the same slice
    elif regime == "huge":
        x *= 1e30
    elif regime == "zero_slices":
        x[0, 128:384] = 0.0
        x[0, 640:768] = 0.0
    else:
        x[0, 512:520] *= 3e4
    check(codes, scales, zeros, 128, "asym", synth.bf16_bits(x.to(torch.bfloat16)))


@pytest.mark.parametrize("M", [1, 3])
def test_rows_split_along_k(M):
    """A row too long for one block (K = 65536 at M = 1) is split along K over two blocks per
    row range; the parts' sums meet in the workspace and the last block adds them in order."""
    N, K, g = 100, 65536, 128
    s = w4.w4a16_gemv_schedule(M, N, K, g, torch.cuda.get_device_properties(0).multi_processor_count)
    assert s["k_parts"] >= 2 and s["workspace_bytes"] > 0
    codes, scales, zeros = quantized("t3", K, N, g, "asym", "one")
    x = synth.normal((M, K), 1.0, 7, 17 + M)
    check(codes, scales, zeros, g, "asym", synth.bf16_bits(x))


@pytest.mark.parametrize("M,K", [(4, 28672), (16, 14336), (5, 4096)])
def test_activation_rows_per_sweep(M, K):
    """Several activation rows per sweep (4 at K <= 14336, 2 at K = 28672) and several
    sweeps over the weights for M > 4."""
    N = 96
    codes, scales, zeros = quantized("t3", K, N, 128, "asym", "one")
    x = synth.normal((M, K), 1.0, 9, M + K)
    check(codes, scales, zeros, 128, "asym", synth.bf16_bits(x))


def test_overlapped_chain_reads_predecessor_output():
    """Three K x K GEMVs back to back with W4_OVERLAP_PREVIOUS, each consuming the previous
    one's bf16 output: the overlapped kernel must read its activations only after its
    predecessor finished. Compared with the oracle's own chain (bf16 between layers). The
    bound is 2e-3 rather than 1e-3: each layer's bf16 rounding of its input can differ from
    the oracle's by one unit where the two fp32/fp64 values straddle a rounding boundary, and
    the next layer carries that difference along, so three layers add up to about twice the
    single-layer bound."""
    K, g = 2048, 128
    qs = []
    for i in range(3):
        W = synth.student_t3_weight(K, K, 9, 950 + i)
        qs.append(oracle.quantize(synth.bf16_bits(W), g, "asym", [1.0], want_chosen=False)[:3])
    x0 = synth.normal((1, K), 1.0, 9, 999)
    # oracle chain
    xb = synth.bf16_bits(x0)
    for codes, scales, zeros in qs:
        y = oracle.gemv_ref(xb, codes, scales, zeros, g, "asym")
        xb = synth.bf16_bits(torch.from_numpy(y).to(torch.float32).to(torch.bfloat16))
    ref = y
    # GPU chain, one workspace shared by the three calls
    ws = w4.alloc_gemv_workspace(K, K, g)
    packs = []
    for codes, scales, zeros in qs:
        p = w4.alloc_packed(K, K, g, w4.W4_LAYOUT_GEMV)
        w4.w4_prepack(to_dev(codes), to_dev(scales.view(np.int16)), to_dev(zeros), K, K, g, "asym",
                      w4.W4_LAYOUT_GEMV, p)
        packs.append(p)
    bufs = [x0.to(cuda())] + [torch.empty(1, K, dtype=torch.bfloat16, device=cuda()) for _ in range(3)]
    torch.cuda.synchronize()
    for rep in range(3):
        for i, p in enumerate(packs):
            w4.w4a16_gemv(bufs[i], 1, p, K, K, g, "asym", bufs[i + 1], w4.W4_OVERLAP_PREVIOUS, ws)
        torch.cuda.synchronize()
        got = bufs[3].float().cpu().numpy().astype(np.float64)
        assert rel_frob(bf16_round(ref), got) <= 2e-3
    assert w4.w4_device_status() == 0


def upload_gemv(codes, scales, zeros, N, K, group, mode):
    packed = w4.alloc_packed(N, K, group, w4.W4_LAYOUT_GEMV)
    w4.w4_prepack(to_dev(codes), to_dev(scales.view(np.int16)), to_dev(zeros) if zeros is not None else None,
                  N, K, group, mode, w4.W4_LAYOUT_GEMV, packed)
    return packed


@pytest.mark.parametrize("M", [1, 3])
def test_grouped_decode_shapes(M):
    """The four decode GEMVs as one grouped launch: every problem against the oracle, both
    output types."""
    probs = []
    for K, N in synth.DECODE_SHAPES:
        codes, scales, zeros = quantized("decode", K, N, 128, "asym", "twenty")
        x_bits = synth.bf16_bits(synth.decode_activation(M, K, 0))
        probs.append((K, N, upload_gemv(codes, scales, zeros, N, K, 128, "asym"), x_bits,
                      oracle.gemv_ref(x_bits, codes, scales, zeros, 128, "asym")))
    xs = [to_dev(p[3].view(np.int16)).view(torch.bfloat16) for p in probs]
    for out_fp32 in (1, 0):
        dt = torch.float32 if out_fp32 else torch.bfloat16
        ys = [torch.full((M, N), float("nan"), dtype=dt, device=cuda()) for K, N, *_ in probs]
        w4.w4a16_gemv_grouped(xs, M, [p[2] for p in probs], [p[1] for p in probs], [p[0] for p in probs], 128,
                              "asym", ys, w4.W4_OUT_FP32 if out_fp32 else 0)
        torch.cuda.synchronize()
        assert w4.w4_device_status() == 0
        for (K, N, _, _, ref), y in zip(probs, ys):
            got = y.double().cpu().numpy()
            assert np.isfinite(got).all()
            if out_fp32:
                assert rel_frob(ref, got) <= 1e-4, (K, N)
            else:
                assert rel_frob(bf16_round(ref), got) <= 1e-3, (K, N)


def test_grouped_ragged_shapes_group_64():
    """Unequal, ragged problems in one group: one row per block for the small ones."""
    M, g = 1, 64
    probs = []
    for N, K in [(77, 320), (5, 4096), (1000, 2048)]:
        codes, scales, zeros = quantized("t3", K, N, g, "asym", "one")
        x_bits = synth.bf16_bits(synth.normal((M, K), 1.0, 3, K + N))
        probs.append((K, N, upload_gemv(codes, scales, zeros, N, K, g, "asym"), x_bits,
                      oracle.gemv_ref(x_bits, codes, scales, zeros, g, "asym")))
    xs = [to_dev(p[3].view(np.int16)).view(torch.bfloat16) for p in probs]
    ys = [torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda()) for K, N, *_ in probs]
    w4.w4a16_gemv_grouped(xs, M, [p[2] for p in probs], [p[1] for p in probs], [p[0] for p in probs], g, "asym",
                          ys, w4.W4_OUT_FP32)
    torch.cuda.synchronize()
    assert w4.w4_device_status() == 0
    for (K, N, _, _, ref), y in zip(probs, ys):
        assert rel_frob(ref, y.double().cpu().numpy()) <= 1e-4, (K, N)


@pytest.mark.parametrize("M", [1, 3])
def test_prefetch_next_decode_chain(M):
    """The four decode GEMVs chained with W4_OVERLAP_PREVIOUS, each naming the next one's
    weights (the last names the first's) for the L2 prefetch: every output against the oracle,
    and bit-identical to the same calls through w4a16_gemv."""
    probs = []
    for K, N in synth.DECODE_SHAPES:
        codes, scales, zeros = quantized("decode", K, N, 128, "asym", "twenty")
        x_bits = synth.bf16_bits(synth.decode_activation(M, K, 0))
        probs.append((K, N, upload_gemv(codes, scales, zeros, N, K, 128, "asym"),
                      to_dev(x_bits.view(np.int16)).view(torch.bfloat16),
                      oracle.gemv_ref(x_bits, codes, scales, zeros, 128, "asym")))
    for out_fp32 in (1, 0):
        dt = torch.float32 if out_fp32 else torch.bfloat16
        flags = w4.W4_OVERLAP_PREVIOUS | (w4.W4_OUT_FP32 if out_fp32 else 0)
        ys = [torch.full((M, N), float("nan"), dtype=dt, device=cuda()) for K, N, *_ in probs]
        plain = [torch.full((M, N), float("nan"), dtype=dt, device=cuda()) for K, N, *_ in probs]
        for rep in range(2):
            for j, (K, N, p, x, _) in enumerate(probs):
                nxt = probs[(j + 1) % len(probs)][2]
                w4.w4a16_gemv_prefetch_next(x, M, p, N, K, 128, "asym", ys[j], flags, None, nxt)
        for j, (K, N, p, x, _) in enumerate(probs):
            w4.w4a16_gemv(x, M, p, N, K, 128, "asym", plain[j], flags, None)
        torch.cuda.synchronize()
        assert w4.w4_device_status() == 0
        for (K, N, _, _, ref), y, yp in zip(probs, ys, plain):
            got = y.double().cpu().numpy()
            assert np.isfinite(got).all()
            assert torch.equal(y, yp), (K, N)
            if out_fp32:
                assert rel_frob(ref, got) <= 1e-4, (K, N)
            else:
                assert rel_frob(bf16_round(ref), got) <= 1e-3, (K, N)


@pytest.mark.parametrize("next_bytes", [0, 8, 16, 4000, 40965, None])
def test_prefetch_next_ranges(next_bytes):
    """Prefetch ranges of every kind (none, below 16 bytes, one 16-byte unit, fewer units than
    blocks, a count that is not a multiple of 16, a whole buffer) on a shape whose rows are
    split along K over several blocks: the result equals w4a16_gemv's bit for bit."""
    N, K, g, M = 100, 65536, 128, 1
    codes, scales, zeros = quantized("t3", K, N, g, "asym", "one")
    p = upload_gemv(codes, scales, zeros, N, K, g, "asym")
    x_bits = synth.bf16_bits(synth.normal((M, K), 1.0, 7, 71))
    x = to_dev(x_bits.view(np.int16)).view(torch.bfloat16)
    other = torch.zeros(1 << 20, dtype=torch.uint8, device=cuda())
    nb = other.numel() if next_bytes is None else next_bytes
    ws = w4.alloc_gemv_workspace(N, K, g)
    y = torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda())
    yp = torch.full((M, N), float("nan"), dtype=torch.float32, device=cuda())
    w4.w4a16_gemv_prefetch_next(x, M, p, N, K, g, "asym", y, w4.W4_OUT_FP32, ws,
                                other if nb else None, nb)
    w4.w4a16_gemv(x, M, p, N, K, g, "asym", yp, w4.W4_OUT_FP32, ws)
    torch.cuda.synchronize()
    assert w4.w4_device_status() == 0
    assert torch.equal(y, yp)
    ref = oracle.gemv_ref(x_bits, codes, scales, zeros, g, "asym")
    assert rel_frob(ref, y.double().cpu().numpy()) <= 1e-4
