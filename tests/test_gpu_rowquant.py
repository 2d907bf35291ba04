"""GPU fp8_row_quant vs the CPU oracle: E4M3 bytes, row scales and group sums must be
bit-identical, and the GEMM's group-sum operand must be the documented bf16 hi/lo split of
the oracle's group sums, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import cuda, gsum_operand, np_of

pytestmark = pytest.mark.gpu


def gpu_row_quant(X, group, op_only=False):
    M, K = X.shape
    Xd = X.to(cuda())
    if group:
        X8, s, G, gop = w4.alloc_row_quant(M, K, group, device=cuda(), group_sums=not op_only)
        gop.fill_(7.0)  # the kernel must write every column, padding included
    else:
        X8 = torch.empty(M, K, dtype=torch.uint8, device=cuda())
        s = torch.empty(M, dtype=torch.float32, device=cuda())
        G = gop = None
    w4.fp8_row_quant(Xd, M, K, group if group else 32, X8, s, G, gop)
    torch.cuda.synchronize()
    op = gop.view(torch.int16).cpu().numpy().view(np.uint16) if gop is not None else None
    return np_of(X8), np_of(s), (np_of(G) if G is not None else None), op


def check(X, group, rows=None, op_only=False):
    gX8, gs, gG, gop = gpu_row_quant(X, group, op_only)
    bits = synth.bf16_bits(X)
    if rows is not None:
        bits = bits[rows]
        gX8, gs = gX8[rows], gs[rows]
        gG = gG[rows] if gG is not None else None
        gop = gop[rows] if gop is not None else None
    X8, s, G = oracle.row_quant(bits, group)
    assert np.array_equal(gs.view(np.uint32), s.view(np.uint32))
    bad = np.argwhere(gX8 != X8)
    assert bad.size == 0, f"{len(bad)} byte mismatches, first {bad[:3].tolist()}"
    if group:
        if not op_only:
            assert np.array_equal(gG.view(np.uint32), G.view(np.uint32))
        assert np.array_equal(gop, gsum_operand(G, X.shape[1], group))


@pytest.mark.parametrize("K", [3840, 15360])
def test_prefill_activations_full_size(K):
    X = synth.prefill_activation(4096, K)
    rows = None if K == 3840 else np.linspace(0, 4095, 512).astype(int)
    check(X, 128, rows)


def test_moe_activations_g32():
    X = synth.moe_activation()
    r = synth.moe_routing()
    Xp = X[r.token_of_row]
    check(Xp, 32, np.linspace(0, Xp.shape[0] - 1, 1024).astype(int))


def test_every_bf16_value():
    """All 65,536 bf16 patterns (finite ones), 512 per row, under several row maxima."""
    pats = np.arange(65536, dtype=np.uint32)
    v = (pats << 16).view(np.float32)
    v = v[np.isfinite(v)]
    v = np.concatenate([v, np.zeros((-v.size) % 512, np.float32)])
    X = torch.from_numpy(v.reshape(-1, 512)).to(torch.bfloat16)
    check(X, 128)


def test_edge_rows():
    K = 256
    rows = [np.zeros(K), np.full(K, 3e-9), np.full(K, -5e-7), np.full(K, 448.0), np.full(K, 1e30),
            np.linspace(-1, 1, K), np.r_[np.ones(K - 1) * 1e-3, 2.0]]
    X = torch.tensor(np.array(rows), dtype=torch.float32).to(torch.bfloat16)
    for g in (32, 64, 128):
        check(X, g)
    check(X, 0)


@pytest.mark.parametrize("M,K", [(1, 16), (3, 48), (2, 2048), (5, 4096 + 32), (2, 16384), (2, 20000 // 16 * 16),
                                 (1, 40960)])
def test_ragged_and_long_rows(M, K):
    X = synth.normal((M, K), 1.0, 2, M + K)
    check(X, 0)
    if K % 32 == 0:
        check(X, 32)
        check(X, 32, op_only=True)
