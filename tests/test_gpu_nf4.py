"""NF4 comparator on the GPU against the oracle: codes and block scales bit for bit, the
GEMV within the W4A16 tolerances (bf16 output against the fp64 result rounded to bf16 at
1e-3, fp32 output at 1e-4: the products level * x are exact in fp32 up to one rounding and
the sums are fp32)."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import bf16_round, cuda, rel_frob

pytestmark = pytest.mark.gpu


def gpu_nf4(W):
    N, K = W.shape
    codes = torch.empty(N, K // 2, dtype=torch.uint8, device=cuda())
    a = torch.empty(N, K // 64, dtype=torch.float32, device=cuda())
    w4.w4_nf4_quantize(W.to(cuda()), N, K, codes, a)
    return codes, a


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
def test_quantize_and_gemv_decode_shapes(K, N):
    W = synth.decode_weight(K, N)
    codes, a = gpu_nf4(W)
    rc, ra = oracle.nf4_quantize(synth.bf16_bits(W))
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(a.cpu().numpy(), ra)
    for M in (1, 4):
        x = synth.decode_activation(M, K)
        ref = oracle.nf4_gemv_ref(synth.bf16_bits(x), rc, ra)
        y32 = torch.empty(M, N, dtype=torch.float32, device=cuda())
        y16 = torch.empty(M, N, dtype=torch.bfloat16, device=cuda())
        w4.w4_nf4_gemv(x.to(cuda()), M, codes, a, N, K, y32, w4.W4_OUT_FP32)
        w4.w4_nf4_gemv(x.to(cuda()), M, codes, a, N, K, y16, 0)
        torch.cuda.synchronize()
        assert rel_frob(ref, y32.double().cpu().numpy()) <= 1e-4
        assert rel_frob(bf16_round(ref), y16.double().cpu().numpy()) <= 1e-3


def test_quantize_edge_blocks():
    K = 256
    rng = np.random.default_rng(9)
    rows = [np.zeros(K), rng.normal(0, 1, K), np.linspace(-1, 1, K), np.full(K, -0.02),
            rng.normal(0, 1e-30, K), np.r_[np.full(K - 1, 1e-3), 7.0]]
    W = torch.tensor(np.array(rows), dtype=torch.float32).to(torch.bfloat16)
    codes, a = gpu_nf4(W)
    rc, ra = oracle.nf4_quantize(synth.bf16_bits(W))
    torch.cuda.synchronize()
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(a.cpu().numpy(), ra)


def test_ragged_rows_and_long_k():
    # the first three take the general kernel; the rest the one-block-per-SM kernel for M = 1
    # and K a multiple of 1024 up to 16384 (single rows, ragged row runs, the longest rows,
    # more rows than 148 blocks of 256 hold)
    for N, K in [(1, 64), (37, 576), (5, 28672), (1, 1024), (149, 2048), (300, 16384), (40000, 1024)]:
        W = synth.student_t3_weight(N, K, 3, N + K)
        codes, a = gpu_nf4(W)
        rc, ra = oracle.nf4_quantize(synth.bf16_bits(W))
        x = synth.normal((1, K), 1.0, 3, K)
        y = torch.full((1, N), float("nan"), dtype=torch.float32, device=cuda())
        w4.w4_nf4_gemv(x.to(cuda()), 1, codes, a, N, K, y, w4.W4_OUT_FP32)
        ref = oracle.nf4_gemv_ref(synth.bf16_bits(x), rc, ra)
        torch.cuda.synchronize()
        assert np.array_equal(codes.cpu().numpy(), rc)
        assert rel_frob(ref, y.double().cpu().numpy()) <= 1e-4
