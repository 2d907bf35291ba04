"""GPU w4a16_gemm_tc (the tensor-core W4A16 for 1 <= M <= 16) vs the CPU oracle's fp64 product
of the dequantized weight, and its W4_LAYOUT_TC prepack vs a numpy re-layout of the canonical
weight.

Tolerances (relative Frobenius), as for w4a16_gemv: bf16 output against the fp64 result
rounded to bf16 at 1e-3, fp32 output against the unrounded result at 1e-4. The kernel's
products of the expanded weights (exact bf16 integers q - 8) with bf16 activations are exact
in fp32; the tensor cores sum 16 of them per step into fp32 accumulators, and the group scale
and the zero-point term are applied in fp32, so the expected error is ~1e-6 relative."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import bf16_round, cuda, rel_frob, to_dev
from test_gpu_gemv import quantized

pytestmark = pytest.mark.gpu


def tc_layout_ref(codes, scales, zeros, N, K, g):
    """W4_LAYOUT_TC written out with numpy from the layout's definition (units of 128 rows x
    max(128, g) k, tile by tile; per unit the code chunks chunk-major then the scales
    group-major)."""
    ks = max(128, g)
    T, NKB = -(-N // 128), -(-K // ks)
    q = np.zeros((T * 128, NKB * ks), np.uint32)
    q[:N, 0:K:2] = codes & 15
    q[:N, 1:K:2] = codes >> 4
    J = K // g
    sc = np.zeros((T * 128, NKB * ks // g), np.uint32)
    z = (zeros.astype(np.int64) & 0xFFFF) if zeros is not None else np.full((N, J), 8)
    sc[:N, :J] = scales.astype(np.uint32) | (z.astype(np.uint32) << 16)
    perm = [0, 2, 4, 6, 1, 3, 5, 7]  # nibble p holds k = perm[p] of its 8
    out = []
    for t in range(T):
        for kb in range(NKB):
            blk = q[t * 128:(t + 1) * 128, kb * ks:(kb + 1) * ks].reshape(128, ks // 32, 4, 8)
            words = np.zeros(blk.shape[:3], np.uint32)
            for p, kk in enumerate(perm):
                words |= blk[..., kk] << np.uint32(4 * p)
            out.append(words.transpose(1, 0, 2).ravel())
            gps = ks // g
            out.append(sc[t * 128:(t + 1) * 128, kb * gps:(kb + 1) * gps].T.ravel())
    return np.concatenate(out)


def upload_tc(codes, scales, zeros, N, K, group, mode):
    packed = w4.alloc_packed(N, K, group, w4.W4_LAYOUT_TC)
    w4.w4_prepack(to_dev(codes), to_dev(scales.view(np.int16)), to_dev(zeros) if zeros is not None else None,
                  N, K, group, mode, w4.W4_LAYOUT_TC, packed)
    return packed


def gpu_tc(packed, N, K, group, mode, x_bits, out_fp32, ws=None):
    M = x_bits.shape[0]
    x = to_dev(x_bits.view(np.int16)).view(torch.bfloat16)
    # NaN-filled, so that an output the kernel does not write cannot pass as a stale value
    y = torch.full((M, N), float("nan"), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=cuda())
    ws = w4.alloc_tc_workspace(N, K, group) if ws is None else ws
    w4.w4a16_gemm_tc(x, M, packed, N, K, group, mode, y, w4.W4_OUT_FP32 if out_fp32 else 0, ws)
    torch.cuda.synchronize()
    assert w4.w4_device_status() == 0
    out = y.float().cpu().numpy().astype(np.float64)
    assert np.isfinite(out).all(), f"unwritten outputs in columns {np.unique(np.nonzero(~np.isfinite(out))[1])[:20]}"
    return out


def check(codes, scales, zeros, group, mode, x_bits):
    N, K = codes.shape[0], codes.shape[1] * 2
    ref = oracle.gemv_ref(x_bits, codes, scales, zeros, group, mode)
    packed = upload_tc(codes, scales, zeros, N, K, group, mode)
    y32 = gpu_tc(packed, N, K, group, mode, x_bits, 1)
    e32 = rel_frob(ref, y32)
    bad = np.nonzero(np.abs(y32 - ref).max(axis=0) > 1e-3 * np.abs(ref).max())[0]
    assert e32 <= 1e-4, (e32, len(bad), bad[:20].tolist())
    y16 = gpu_tc(packed, N, K, group, mode, x_bits, 0)
    e16 = rel_frob(bf16_round(ref), y16)
    assert e16 <= 1e-3, e16
    return e32, e16


@pytest.mark.parametrize("group,mode", [(32, "sym"), (64, "asym"), (128, "asym"), (256, "sym")])
def test_layout_bytes(group, mode):
    N, K = 200, 768  # two tiles (the second ragged); K not a multiple of 512
    codes, scales, zeros = quantized("t3", K, N, group, mode, "one")
    packed = upload_tc(codes, scales, zeros, N, K, group, mode)
    torch.cuda.synchronize()
    got = packed.cpu().numpy().view(np.uint32)
    want = tc_layout_ref(codes, scales, zeros, N, K, group)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
@pytest.mark.parametrize("M", synth.DECODE_M)
def test_decode_sweep_full_size(K, N, M):
    codes, scales, zeros = quantized("decode", K, N, 128, "asym", "twenty")
    x = synth.decode_activation(M, K)
    check(codes, scales, zeros, 128, "asym", synth.bf16_bits(x))


@pytest.mark.parametrize("M", [1, 2, 3, 5, 9, 16])
@pytest.mark.parametrize("group,mode", [(32, "sym"), (64, "asym"), (128, "asym"), (128, "sym"), (256, "asym")])
def test_ragged(M, group, mode):
    N = 77                              # one ragged tile
    K = 320 if group < 128 else (384 if group == 128 else 768)  # k-blocks with zero padding
    codes, scales, zeros = quantized("t3", K, N, group, mode, "twenty")
    x = synth.normal((M, K), 1.0, 4, 31 * M + group)
    check(codes, scales, zeros, group, mode, synth.bf16_bits(x))


@pytest.mark.parametrize("N,K,M", [(1, 32, 1), (8, 128, 3), (9, 64, 16), (129, 4096, 4), (300, 2048, 7)])
def test_small_and_shared_tiles(N, K, M):
    """Tiny problems (one CTA per k-block of one tile: every tile shared by many CTAs) and
    tiles split across CTAs at arbitrary k-blocks."""
    g = 32 if K < 128 else 128
    codes, scales, zeros = quantized("t3", K, N, g, "asym", "one")
    x = synth.normal((M, K), 1.0, 5, N + K + M)
    check(codes, scales, zeros, g, "asym", synth.bf16_bits(x))


def test_extreme_zero_points():
    """One-signed blocks make |z| large; the zero-point term (z - 8) X_j carries them exactly
    to fp32 rounding."""
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


def test_one_hot_columns_exact():
    """x = unit vectors: each output row is one column of the dequantized weight, which the
    kernel must reproduce exactly (one nonzero product per group, scale applied once)."""
    K, N = 512, 200
    codes, scales, zeros = quantized("t3", K, N, 128, "asym", "one")
    cols = [0, 131, 300, 511]
    x = np.zeros((len(cols), K), np.float32)
    for i, c in enumerate(cols):
        x[i, c] = 1.0
    xb = synth.bf16_bits(torch.from_numpy(x).to(torch.bfloat16))
    packed = upload_tc(codes, scales, zeros, N, K, 128, "asym")
    y = gpu_tc(packed, N, K, 128, "asym", xb, 1)
    Wd = oracle.dequantize(codes, scales, zeros, 128, "asym")
    for i, c in enumerate(cols):
        assert np.array_equal(y[i], Wd[:, c].astype(np.float32).astype(np.float64))


def test_deterministic_and_workspace_clean():
    """Two calls give the same bits, and the workspace's counters are zero after each."""
    K, N, M, g = 4096, 1024, 4, 128
    codes, scales, zeros = quantized("decode", K, N, g, "asym", "twenty")
    x = synth.bf16_bits(synth.decode_activation(M, K))
    packed = upload_tc(codes, scales, zeros, N, K, g, "asym")
    ws = w4.alloc_tc_workspace(N, K, g)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    part_bytes = sms * 2 * 128 * 16 * 4
    a = gpu_tc(packed, N, K, g, "asym", x, 1, ws)
    assert int(ws[part_bytes:].count_nonzero()) == 0
    b = gpu_tc(packed, N, K, g, "asym", x, 1, ws)
    assert np.array_equal(a, b)
    assert int(ws[part_bytes:].count_nonzero()) == 0


def test_overlapped_chain_reads_predecessor_output():
    """Three K x K layers back to back with W4_OVERLAP_PREVIOUS at M = 4, each consuming the
    previous one's bf16 output (bound 2e-3: see the same test of w4a16_gemv)."""
    K, g, M = 2048, 128, 4
    qs = []
    for i in range(3):
        W = synth.student_t3_weight(K, K, 9, 960 + i)
        qs.append(oracle.quantize(synth.bf16_bits(W), g, "asym", [1.0], want_chosen=False)[:3])
    x0 = synth.normal((M, K), 1.0, 9, 998)
    xb = synth.bf16_bits(x0)
    for codes, scales, zeros in qs:
        y = oracle.gemv_ref(xb, codes, scales, zeros, g, "asym")
        xb = synth.bf16_bits(torch.from_numpy(y).to(torch.float32).to(torch.bfloat16))
    ref = y
    ws = w4.alloc_tc_workspace(K, K, g)
    packs = [upload_tc(c, s, z, K, K, g, "asym") for c, s, z in qs]
    bufs = [x0.to(cuda())] + [torch.empty(M, K, dtype=torch.bfloat16, device=cuda()) for _ in range(3)]
    torch.cuda.synchronize()
    for rep in range(3):
        for i, p in enumerate(packs):
            w4.w4a16_gemm_tc(bufs[i], M, p, K, K, g, "asym", bufs[i + 1], w4.W4_OVERLAP_PREVIOUS, ws)
        torch.cuda.synchronize()
        got = bufs[3].float().cpu().numpy().astype(np.float64)
        assert rel_frob(bf16_round(ref), got) <= 2e-3
    assert w4.w4_device_status() == 0
