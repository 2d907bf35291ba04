"""GPU w4a8_gemm / w4a8_grouped_gemm vs the CPU oracle's fp64 product of the two
dequantized operands (E4M3 activations times row scale, INT4 weights times group scale).

Gate: relative Frobenius error <= 2e-2 (the required bound). A tighter bound is also
asserted because the tensor-core operands are exact. For groups of 64 and 128 the expanded
codes are exact small integers in E4M3, the activations are the E4M3 codes themselves, and
what remains is fp32 accumulation (~1e-6) and the bf16 hi/lo zero-point term (~2^-16 of that
term). For groups of 32 the dequantized weight (q - z) s is split exactly into two fp16
parts and the E4M3 activations are exact in fp16, so only fp32 accumulation remains. For
bf16 output there is one more rounding (<= 2^-9 relative per element): fp32 output must be
within 1e-4 and bf16 output within 4e-3."""
import functools

import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import cuda, gsum_operand, np_of, rel_frob, to_dev

pytestmark = pytest.mark.gpu

TOL_REQUIRED = 2e-2
TOL_F32 = 1e-4
TOL_BF16 = 4e-3


def upload_weight(codes, scales, zeros, N, K, group, mode, copies=1):
    nbytes = w4.w4_prepack_bytes(N, K, group, w4.W4_LAYOUT_GEMM)
    packed = torch.empty(copies * nbytes, dtype=torch.uint8, device=cuda())
    for e in range(copies):
        c = to_dev(codes[e] if copies > 1 else codes)
        s = to_dev((scales[e] if copies > 1 else scales).view(np.int16))
        z = None if zeros is None else to_dev(zeros[e] if copies > 1 else zeros)
        w4.w4_prepack(c, s, z, N, K, group, mode, w4.W4_LAYOUT_GEMM, packed[e * nbytes:])
    return packed


def split_path(group):
    """Groups 32 and 256 run the split-weight fp16 path, which takes the fp16 copy of the E4M3
    activations (and neither the codes nor the group-sum operand)."""
    return group in (32, 256)


def x16_of(X8):
    """The fp16 copy of E4M3 codes (exact), as fp8_row_quant writes it."""
    return to_dev(X8).view(torch.float8_e4m3fn).to(torch.float16)


def gemm_operands(X8, G, K, group):
    if split_path(group):
        return None, None, x16_of(X8)
    return to_dev(X8), to_dev(gsum_operand(G, K, group)), None


def gpu_gemm(X8, s_a, G, packed, N, K, group, mode, out_fp32, ws=None):
    M = X8.shape[0]
    Y = torch.empty(M, N, dtype=torch.float32 if out_fp32 else torch.bfloat16, device=cuda())
    x8, gop, x16 = gemm_operands(X8, G, K, group)
    w4.w4a8_gemm(x8, to_dev(s_a), gop, M, packed, N, K, group, mode, Y, out_fp32, ws, X16=x16)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64)


def split_workspace(M, N, K, group):
    """Zero-filled workspace when this shape's last wave is split along K on this GPU, else None."""
    return w4.alloc_gemm_workspace(M, N, K, group, device=cuda())


def check_split_run(X8, s_a, G, packed, N, K, group, mode, ref, rows=None):
    """With a workspace: the split schedule within the same bounds, bit-identical on a second
    call (the first left the arrival counters at zero), counters zero afterwards."""
    M = X8.shape[0]
    ws = split_workspace(M, N, K, group)
    if ws is None:
        return False
    y32 = gpu_gemm(X8, s_a, G, packed, N, K, group, mode, 1, ws)
    y16 = gpu_gemm(X8, s_a, G, packed, N, K, group, mode, 0, ws)
    y32b = gpu_gemm(X8, s_a, G, packed, N, K, group, mode, 1, ws)
    assert np.array_equal(y32, y32b)
    sel = slice(None) if rows is None else rows
    check_errors(ref, y32[sel], y16[sel])
    sched = w4.w4a8_gemm_schedule(M, N, K, group, torch.cuda.get_device_properties(0).multi_processor_count)
    counters = ws[ws.numel() - sched["split_tiles"] * 32:]
    assert int(counters.count_nonzero()) == 0
    assert w4.w4_device_status() == 0
    return True


def check_errors(ref, y32, y16):
    e32, e16 = rel_frob(ref, y32), rel_frob(ref, y16)
    assert e32 <= TOL_REQUIRED and e16 <= TOL_REQUIRED, (e32, e16)
    assert e32 <= TOL_F32, e32
    assert e16 <= TOL_BF16, e16
    return e32, e16


def run_dense(M, N, K, group, mode, seed=0, grid=(1.0,), outlier_cols=8):
    W = synth.student_t3_weight(N, K, seed, 800 + N + K)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), group, mode, list(grid), want_chosen=False)
    X = synth.outlier_activation(M, K, outlier_cols, 20.0, seed, 850 + M)
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), group)
    ref = oracle.w4a8_ref_dense(X8, s_a, codes, scales, zeros, group, mode)
    packed = upload_weight(codes, scales, zeros, N, K, group, mode)
    y32 = gpu_gemm(X8, s_a, G, packed, N, K, group, mode, 1)
    y16 = gpu_gemm(X8, s_a, G, packed, N, K, group, mode, 0)
    errs = check_errors(ref, y32, y16)
    check_split_run(X8, s_a, G, packed, N, K, group, mode, ref)
    return errs


@pytest.mark.parametrize("group", [32, 64, 128, 256])
@pytest.mark.parametrize("mode", ["asym", "sym"])
def test_one_tile(group, mode):
    run_dense(128, 128, 256, group, mode)


@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (7, 77, 160), (129, 200, 384), (300, 256, 2880),
                                   (256, 384, 1024), (1000, 130, 640)])
def test_ragged_shapes(M, N, K):
    g = 32 if K % 64 else 64
    run_dense(M, N, K, g, "asym")
    run_dense(M, N, K, 32, "sym")


def test_long_k_many_groups():
    run_dense(256, 256, 15360, 128, "asym")


@pytest.mark.parametrize("M,N,K,group,mode", [(256, 256, 15360, 128, "asym"), (300, 256, 2880, 64, "sym"),
                                              (300, 1500, 4096, 64, "asym"), (40, 640, 8192, 128, "asym")])
def test_split_schedule_is_used(M, N, K, group, mode):
    """Shapes whose tiles are split along K on a 148-SM B200 (two long tiles over 16 blocks;
    ragged K; ragged N with 24 tiles; a single token tile): the split result is checked
    against the oracle inside run_dense; here also that the split really happened."""
    assert split_workspace(M, N, K, group) is not None
    run_dense(M, N, K, group, mode)


@functools.lru_cache(maxsize=None)
def prefill_case(K, N):
    W = synth.prefill_weight(K, N)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), 128, "asym", [1.0], want_chosen=False)
    X = synth.prefill_activation(synth.PREFILL_M, K)
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), 128)
    return codes, scales, zeros, X8, s_a, G


@pytest.mark.parametrize("K,N", synth.PREFILL_SHAPES)
def test_prefill_full_size_sampled_rows(K, N):
    """M=4096 prefill at full size; the oracle evaluates 48 token rows against every
    output column (fp64 product of the dequantized operands)."""
    codes, scales, zeros, X8, s_a, G = prefill_case(K, N)
    packed = upload_weight(codes, scales, zeros, N, K, 128, "asym")
    y32 = gpu_gemm(X8, s_a, G, packed, N, K, 128, "asym", 1)
    y16 = gpu_gemm(X8, s_a, G, packed, N, K, 128, "asym", 0)
    # the last token rows lie in the tiles that the split schedule divides along K
    rows = np.unique(np.r_[np.arange(8), np.linspace(0, 4095, 32).astype(int), np.arange(3840, 3848),
                           np.arange(4088, 4096)])
    Wd = oracle.dequantize(codes, scales, zeros, 128, "asym")
    A = oracle.e4m3_decode(X8[rows]).astype(np.float64) * s_a[rows, None].astype(np.float64)
    ref = A @ Wd.T
    check_errors(ref, y32[rows], y16[rows])
    check_split_run(X8, s_a, G, packed, N, K, 128, "asym", ref, rows)


def test_pipeline_gpu_rowquant_then_gemm():
    """bf16 X -> GPU fp8_row_quant -> GPU w4a8_gemm, against the oracle's whole chain."""
    M, N, K, g = 512, 384, 1536, 128
    W = synth.student_t3_weight(N, K, 1, 77)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), g, "asym", synth.clip_grid_20(), want_chosen=False)
    X = synth.outlier_activation(M, K, 8, 20.0, 1, 78)
    X8r, s_ar, _ = oracle.row_quant(synth.bf16_bits(X), g)
    ref = oracle.w4a8_ref_dense(X8r, s_ar, codes, scales, zeros, g, "asym")
    packed = upload_weight(codes, scales, zeros, N, K, g, "asym")
    Xd = X.to(cuda())
    X8, s_a, _, gop = w4.alloc_row_quant(M, K, g, device=cuda(), group_sums=False)
    w4.fp8_row_quant(Xd, M, K, g, X8, s_a, None, gop)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=cuda())
    w4.w4a8_gemm(X8, s_a, gop, M, packed, N, K, g, "asym", Y, 0)
    torch.cuda.synchronize()
    e = rel_frob(ref, Y.float().cpu().numpy())
    assert e <= TOL_BF16, e


# ------------------------------------------------------------------ grouped (MoE)

def grouped_case(E, N, K, g, rows_per_expert, seed=0):
    codes, scales, zeros = [], [], []
    for e in range(E):
        W = synth.normal((N, K), 0.02, seed, 300 + e)
        c, s, z, _ = oracle.quantize(synth.bf16_bits(W), g, "asym", [1.0], want_chosen=False)
        codes.append(c); scales.append(s); zeros.append(z)
    codes, scales, zeros = np.stack(codes), np.stack(scales), np.stack(zeros)
    off = np.zeros(E + 1, np.int32)
    off[1:] = np.cumsum(rows_per_expert)
    M = int(off[-1])
    X = synth.normal((M, K), 1.0, seed, 399)
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), g)
    return codes, scales, zeros, off, X8, s_a, G


def gpu_grouped(codes, scales, zeros, off, X8, s_a, G, N, K, g):
    E = codes.shape[0]
    M = X8.shape[0]
    packed = upload_weight(codes, scales, zeros, N, K, g, "asym", copies=E)
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=cuda())
    x8, gop, x16 = gemm_operands(X8, G, K, g)
    w4.w4a8_grouped_gemm(x8, to_dev(s_a), gop, to_dev(off), E, M, packed, N, K, g, "asym", Y, X16=x16)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64)


def expert_of_rows(off):
    return np.repeat(np.arange(len(off) - 1, dtype=np.int32), np.diff(off))


def test_grouped_small_with_empty_expert():
    N, K, g = 256, 2880, 32
    rows = [5, 0, 200, 131]
    codes, scales, zeros, off, X8, s_a, G = grouped_case(4, N, K, g, rows)
    Y = gpu_grouped(codes, scales, zeros, off, X8, s_a, G, N, K, g)
    ex = expert_of_rows(off)
    mm, nn = np.meshgrid(np.arange(X8.shape[0]), np.arange(N), indexing="ij")
    ref = oracle.w4a8_ref_pairs(X8, s_a, codes, scales, zeros, g, "asym", mm.ravel(), nn.ravel(), ex)
    e = rel_frob(ref, Y.ravel())
    assert e <= TOL_BF16, e


@pytest.mark.parametrize("kind", ["gate_up", "down"])
def test_moe_full_size_sampled(kind):
    """32 experts, 4096 tokens routed top-4 (16,384 rows), K=2880, group 32: every expert's
    weight quantized by the oracle; 8192 sampled outputs compared."""
    c = synth.MOE
    N = c["N_gate_up"] if kind == "gate_up" else c["N_down"]
    K, g, E = c["K"], c["group"], c["E"]
    codes, scales, zeros = [], [], []
    for e in range(E):
        W = synth.moe_weight(kind, e)
        cc, ss, zz, _ = oracle.quantize(synth.bf16_bits(W), g, "asym", [1.0], want_chosen=False)
        codes.append(cc); scales.append(ss); zeros.append(zz)
    codes, scales, zeros = np.stack(codes), np.stack(scales), np.stack(zeros)
    r = synth.moe_routing()
    X = synth.moe_activation()[r.token_of_row]
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), g)
    off = r.expert_row_offsets.numpy()
    Y = gpu_grouped(codes, scales, zeros, off, X8, s_a, G, N, K, g)
    rng = np.random.default_rng(0)
    mm = rng.integers(0, X8.shape[0], 8192)
    nn = rng.integers(0, N, 8192)
    ref = oracle.w4a8_ref_pairs(X8, s_a, codes, scales, zeros, g, "asym", mm, nn, expert_of_rows(off))
    e = rel_frob(ref, Y[mm, nn])
    assert e <= TOL_BF16, e


def test_no_device_status_after_gemms():
    assert w4.w4_device_status() == 0


def test_extreme_zero_points():
    """One-signed blocks give zero points far outside [0, 15]; the zero-point term (through
    the activation group sums) must stay within the same tolerances."""
    rng = np.random.default_rng(4)
    M, N, K, g = 256, 128, 512, 32
    W = rng.normal(0, 0.02, (N, K))
    blocks = W.reshape(N, K // g, g)
    pick = rng.integers(0, 3, (N, K // g))
    blocks[pick == 1] = 1.0 + rng.uniform(0, 0.02, (int((pick == 1).sum()), g))
    blocks[pick == 2] = -3.0 - rng.uniform(0, 0.05, (int((pick == 2).sum()), g))
    bits = synth.bf16_bits(torch.tensor(blocks.reshape(N, K), dtype=torch.float32).to(torch.bfloat16))
    codes, scales, zeros, _ = oracle.quantize(bits, g, "asym", synth.clip_grid_20(), want_chosen=False)
    assert np.abs(zeros).max() > 241
    X = synth.outlier_activation(M, K, 4, 20.0, 0, 5)
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), g)
    ref = oracle.w4a8_ref_dense(X8, s_a, codes, scales, zeros, g, "asym")
    packed = upload_weight(codes, scales, zeros, N, K, g, "asym")
    check_errors(ref, gpu_gemm(X8, s_a, G, packed, N, K, g, "asym", 1), gpu_gemm(X8, s_a, G, packed, N, K, g, "asym", 0))


def test_persistent_tiles_with_long_zero_point_tail():
    """More tiles than SMs, each with K = 11520 (90 groups -> 9 zero-point pseudo-stages, more
    than the 4-slot ring): every pipeline role must stay in lockstep with the ring across
    tiles. 32 sampled token rows against every output column."""
    M, N, K, g = 256, 20480, 11520, 128
    W = synth.normal((N, K), 0.02, 2, 31)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), g, "asym", [1.0], want_chosen=False)
    X = synth.outlier_activation(M, K, 8, 20.0, 2, 32)
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), g)
    packed = upload_weight(codes, scales, zeros, N, K, g, "asym")
    y32 = gpu_gemm(X8, s_a, G, packed, N, K, g, "asym", 1)
    y16 = gpu_gemm(X8, s_a, G, packed, N, K, g, "asym", 0)
    rows = np.linspace(0, M - 1, 32).astype(int)
    Wd = oracle.dequantize(codes, scales, zeros, g, "asym")
    A = oracle.e4m3_decode(X8[rows]).astype(np.float64) * s_a[rows, None].astype(np.float64)
    check_errors(A @ Wd.T, y32[rows], y16[rows])
    assert w4.w4_device_status() == 0
    # 160 tiles on 148 SMs: one whole wave, then 12 tiles split over 96 blocks, 9 zero-point
    # pseudo-stages on the segment that ends each split tile
    assert check_split_run(X8, s_a, G, packed, N, K, g, "asym", A @ Wd.T, rows)


@pytest.mark.parametrize("group", [32, 256])
def test_split_path_persistent_odd_weight_tiles(group):
    """Split-weight path with more tiles than SMs: 4001 tokens (16 token tiles of 256, the last
    holding 161 rows) x 1400 outputs (11 weight tiles of 128, the last holding 120 rows) is 176
    tiles, so some CTAs run two and both TMEM accumulators are used. K = 512. 64 sampled token
    rows (the tile edges among them) against every output column."""
    M, N, K = 4001, 1400, 512
    W = synth.student_t3_weight(N, K, 3, 41)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), group, "asym", [1.0], want_chosen=False)
    X = synth.outlier_activation(M, K, 8, 20.0, 3, 42)
    X8, s_a, G = oracle.row_quant(synth.bf16_bits(X), group)
    packed = upload_weight(codes, scales, zeros, N, K, group, "asym")
    y32 = gpu_gemm(X8, s_a, G, packed, N, K, group, "asym", 1)
    y16 = gpu_gemm(X8, s_a, G, packed, N, K, group, "asym", 0)
    rows = np.unique(np.concatenate([np.linspace(0, M - 1, 60).astype(int), [255, 256, 3839, 3840, 4000]]))
    Wd = oracle.dequantize(codes, scales, zeros, group, "asym")
    A = oracle.e4m3_decode(X8[rows]).astype(np.float64) * s_a[rows, None].astype(np.float64)
    check_errors(A @ Wd.T, y32[rows], y16[rows])
    assert w4.w4_device_status() == 0
