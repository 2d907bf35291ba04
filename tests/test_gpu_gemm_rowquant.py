"""GPU w4a8_gemm_rowquant (row quant and W4A8 GEMM in one launch, from bf16 activations).

The one-launch path must compute exactly what the two-launch path computes
(fp8_row_quant, then w4a8_gemm with a workspace): the E4M3 rows, row scales and group-sum
operand it leaves in its workspace are compared bit for bit with fp8_row_quant's outputs
and with the oracle's row quant ("Four-bit inference ... Tahoma", Achievement 2), and the
output Y bit for bit with the two-launch Y. Y is also checked against the oracle's fp64
product of the dequantized operands with the bounds of the W4A8 GEMM tests (fp32 output
1e-4, bf16 output 4e-3, required 2e-2)."""
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


def packed_weight(N, K, group, mode, seed):
    W = synth.student_t3_weight(N, K, seed, 900 + N + K)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), group, mode, [1.0], want_chosen=False)
    packed = torch.empty(w4.w4_prepack_bytes(N, K, group, w4.W4_LAYOUT_GEMM), dtype=torch.uint8, device=cuda())
    w4.w4_prepack(to_dev(codes), to_dev(scales.view(np.int16)), None if zeros is None else to_dev(zeros),
                  N, K, group, mode, w4.W4_LAYOUT_GEMM, packed)
    return packed, codes, scales, zeros


def two_launch(Xd, M, packed, N, K, group, mode, out_fp32):
    """fp8_row_quant then w4a8_gemm with a (zero-filled) split workspace."""
    X8, sa, _, gop = w4.alloc_row_quant(M, K, group, device=cuda(), group_sums=False)
    w4.fp8_row_quant(Xd, M, K, group, X8, sa, None, gop)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=cuda())
    w4.w4a8_gemm(X8, sa, gop, M, packed, N, K, group, mode, Y, out_fp32,
                 w4.alloc_gemm_workspace(M, N, K, group, device=cuda()))
    torch.cuda.synchronize()
    return Y, X8, sa, gop


def one_launch(Xd, M, packed, N, K, group, mode, out_fp32, ws):
    Y = torch.full((M, N), float("nan"), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=cuda())
    w4.w4a8_gemm_rowquant(Xd, M, packed, N, K, group, mode, Y, out_fp32, ws)
    torch.cuda.synchronize()
    return Y


def workspace_rows(ws, M, N, K, group):
    """The E4M3 rows, row scales and group-sum operand the call left in its workspace."""
    lay = w4.w4a8_gemm_rowquant_layout(M, N, K, group)
    cols = w4.w4a8_gsum_op_cols(K, group)
    X8 = ws[lay["X_e4m3"]:lay["X_e4m3"] + M * K].view(M, K)
    sa = ws[lay["row_scale"]:lay["row_scale"] + 4 * M].view(torch.float32)
    gop = ws[lay["gsum_op"]:lay["gsum_op"] + 2 * M * cols].view(torch.int16).view(M, cols)
    return X8, sa, gop


def check_same_rows(ws, M, N, K, group, X8, sa, gop):
    a8, asa, agop = workspace_rows(ws, M, N, K, group)
    assert torch.equal(a8, X8)
    assert torch.equal(asa.view(torch.int32), sa.view(torch.int32))
    assert torch.equal(agop, gop.view(torch.int16))


def check_oracle(X, codes, scales, zeros, group, mode, ws, M, N, K, y32, y16):
    """Workspace rows bit-exact against the oracle's row quant; outputs within the W4A8 bounds
    of the oracle's fp64 product."""
    X8o, s_ao, Go = oracle.row_quant(synth.bf16_bits(X), group)
    a8, asa, agop = workspace_rows(ws, M, N, K, group)
    assert np.array_equal(np_of(a8), X8o)
    assert np.array_equal(np_of(asa).view(np.uint32), np.asarray(s_ao, np.float32).view(np.uint32))
    assert np.array_equal(np_of(agop).view(np.uint16), gsum_operand(Go, K, group))
    ref = oracle.w4a8_ref_dense(X8o, s_ao, codes, scales, zeros, group, mode)
    e32 = rel_frob(ref, np_of(y32.float()))
    e16 = rel_frob(ref, np_of(y16.float()))
    assert e32 <= TOL_REQUIRED and e16 <= TOL_REQUIRED, (e32, e16)
    assert e32 <= TOL_F32, e32
    assert e16 <= TOL_BF16, e16


# (M, N, K, group, mode): one tile; a single token row; ragged M, N and K; many token tiles
# with a ragged tail; shapes whose last wave is split along K on 148 SMs; a long K; rows longer
# than half the kernel's shared-memory ring (K = 65536), which are not staged through it but
# streamed by warps (the token tiles that the first tiles read first, the rest while the GEMM
# runs)
CASES = [(128, 128, 256, 128, "asym"), (1, 128, 128, 128, "asym"), (7, 77, 192, 64, "sym"),
         (129, 200, 384, 128, "asym"), (1000, 130, 640, 128, "asym"), (300, 256, 2880, 64, "sym"),
         (300, 1500, 4096, 64, "asym"), (40, 640, 8192, 128, "asym"), (256, 256, 15360, 128, "asym"),
         (600, 256, 65536, 128, "asym")]


@pytest.mark.parametrize("M,N,K,group,mode", CASES)
def test_one_launch_equals_two_launches_and_oracle(M, N, K, group, mode):
    packed, codes, scales, zeros = packed_weight(N, K, group, mode, 3)
    X = synth.outlier_activation(M, K, 8, 20.0, 3, 910 + M)
    Xd = X.to(cuda())
    ws = w4.alloc_gemm_rowquant_workspace(M, N, K, group, device=cuda())
    ys = {}
    for out_fp32 in (1, 0):
        Yr, X8, sa, gop = two_launch(Xd, M, packed, N, K, group, mode, out_fp32)
        Y = one_launch(Xd, M, packed, N, K, group, mode, out_fp32, ws)
        assert torch.equal(Y, Yr)
        check_same_rows(ws, M, N, K, group, X8, sa, gop)
        ys[out_fp32] = Y
    check_oracle(X, codes, scales, zeros, group, mode, ws, M, N, K, ys[1], ys[0])
    assert w4.w4_device_status() == 0


def test_workspace_reuse_with_new_activations():
    """Three calls on one workspace, the activations changing between them: each call's rows
    and output are its own (the row counts of the previous call do not let a tile read stale rows)."""
    M, N, K, group = 1000, 384, 3840, 128
    packed, *_ = packed_weight(N, K, group, "asym", 4)
    ws = w4.alloc_gemm_rowquant_workspace(M, N, K, group, device=cuda())
    ws.fill_(0xA5)  # no initial contents are needed
    for i in range(3):
        Xd = synth.outlier_activation(M, K, 8, 20.0, 4, 920 + i).to(cuda())
        Yr, X8, sa, gop = two_launch(Xd, M, packed, N, K, group, "asym", 0)
        Y = one_launch(Xd, M, packed, N, K, group, "asym", 0, ws)
        assert torch.equal(Y, Yr)
        check_same_rows(ws, M, N, K, group, X8, sa, gop)
    assert w4.w4_device_status() == 0


def test_special_rows():
    """An all-zero row (scale 1e-8 / 448, zero codes, zero output), a row at the bf16 maximum,
    and rows holding an infinity or a NaN (IEEE division, as fp8_row_quant): codes and scales
    bit for bit; the outputs of the finite rows bit for bit."""
    M, N, K, group = 300, 256, 1024, 64
    packed, *_ = packed_weight(N, K, group, "asym", 5)
    X = synth.outlier_activation(M, K, 8, 20.0, 5, 930)
    X[3] = 0.0
    X[17, 5] = 3.3895313892515355e38  # bf16 max
    X[200, 9] = float("inf")
    X[201, 11] = float("nan")
    Xd = X.to(cuda())
    ws = w4.alloc_gemm_rowquant_workspace(M, N, K, group, device=cuda())
    Yr, X8, sa, gop = two_launch(Xd, M, packed, N, K, group, "asym", 1)
    Y = one_launch(Xd, M, packed, N, K, group, "asym", 1, ws)
    check_same_rows(ws, M, N, K, group, X8, sa, gop)
    finite = [m for m in range(M) if m not in (200, 201)]
    assert torch.equal(Y[finite], Yr[finite])
    assert int(torch.count_nonzero(Y[3])) == 0


@pytest.mark.parametrize("K,N", synth.PREFILL_SHAPES)
def test_prefill_full_size(K, N):
    """M = 4096 prefill at full size, in the launch configuration the benchmark times: the
    one-launch Y equals the two-launch Y bit for bit (that path is checked against the oracle
    at this size by the W4A8 GEMM tests), and sampled rows of the workspace equal the oracle's
    row quant of those rows."""
    M, group = synth.PREFILL_M, 128
    W = synth.prefill_weight(K, N)
    codes, scales, zeros, _ = oracle.quantize(synth.bf16_bits(W), group, "asym", [1.0], want_chosen=False)
    packed = torch.empty(w4.w4_prepack_bytes(N, K, group, w4.W4_LAYOUT_GEMM), dtype=torch.uint8, device=cuda())
    w4.w4_prepack(to_dev(codes), to_dev(scales.view(np.int16)), to_dev(zeros), N, K, group, "asym",
                  w4.W4_LAYOUT_GEMM, packed)
    X = synth.prefill_activation(M, K)
    Xd = X.to(cuda())
    ws = w4.alloc_gemm_rowquant_workspace(M, N, K, group, device=cuda())
    Yr, X8, sa, gop = two_launch(Xd, M, packed, N, K, group, "asym", 0)
    Y = one_launch(Xd, M, packed, N, K, group, "asym", 0, ws)
    assert torch.equal(Y, Yr)
    check_same_rows(ws, M, N, K, group, X8, sa, gop)
    rows = np.unique(np.r_[np.arange(4), np.linspace(0, M - 1, 24).astype(int), np.arange(M - 4, M)])
    X8o, s_ao, Go = oracle.row_quant(synth.bf16_bits(X[torch.from_numpy(rows)]), group)
    a8, asa, agop = workspace_rows(ws, M, N, K, group)
    assert np.array_equal(np_of(a8)[rows], X8o)
    assert np.array_equal(np_of(asa)[rows].view(np.uint32), np.asarray(s_ao, np.float32).view(np.uint32))
    assert np.array_equal(np_of(agop)[rows].view(np.uint16), gsum_operand(Go, K, group))
    assert w4.w4_device_status() == 0


def packed_weight_gpu(N, K, group, seed):
    """A prepacked weight quantized on the GPU (its quantizer is bit-exact against the oracle
    in the quantizer tests); the comparison below is between two paths on the same weight."""
    dev = cuda()
    W = synth.normal((N, K), 0.02, seed, 960).to(dev)
    codes, scales, zeros, _ = w4.alloc_quantized(N, K, group, "asym", device=dev, chosen=False)
    w4.w4_quantize(W, N, K, group, "asym", [1.0], codes, scales, zeros, None)
    p = w4.alloc_packed(N, K, group, w4.W4_LAYOUT_GEMM, device=dev)
    w4.w4_prepack(codes, scales, zeros, N, K, group, "asym", w4.W4_LAYOUT_GEMM, p)
    return p


@pytest.mark.parametrize("M,N,K", [(2048, 8192, 1024), (2048, 6144, 65536)])
def test_rows_quantized_while_the_gemm_runs(M, N, K):
    """Shapes with more waves of tiles than the rows quantized before the GEMM starts cover:
    the rest of the rows come from two warps per block while the tiles run. At K = 1024 the
    first rows are staged through the shared-memory ring (2048 x 8192: 512 whole tiles, rows
    from 1280 on in the background); at K = 65536 they are streamed by warps and the last wave
    is split along K (2048 x 6144: 384 tiles, rows 1024 to 1535 in the background). Y, codes,
    scales and group-sum operand equal the two-launch path's bit for bit; sampled rows of the
    workspace equal the oracle's row quant."""
    group = 128
    packed = packed_weight_gpu(N, K, group, 6)
    X = synth.outlier_activation(M, K, 8, 20.0, 6, 940)
    Xd = X.to(cuda())
    ws = w4.alloc_gemm_rowquant_workspace(M, N, K, group, device=cuda())
    Yr, X8, sa, gop = two_launch(Xd, M, packed, N, K, group, "asym", 0)
    Y = one_launch(Xd, M, packed, N, K, group, "asym", 0, ws)
    assert torch.equal(Y, Yr)
    check_same_rows(ws, M, N, K, group, X8, sa, gop)
    rows = np.unique(np.r_[0, 255, 256, np.linspace(0, M - 1, 12).astype(int), M - 1])
    X8o, s_ao, Go = oracle.row_quant(synth.bf16_bits(X[torch.from_numpy(rows)]), group)
    a8, asa, agop = workspace_rows(ws, M, N, K, group)
    assert np.array_equal(np_of(a8)[rows], X8o)
    assert np.array_equal(np_of(asa)[rows].view(np.uint32), np.asarray(s_ao, np.float32).view(np.uint32))
    assert np.array_equal(np_of(agop)[rows].view(np.uint16), gsum_operand(Go, K, group))
    assert w4.w4_device_status() == 0
