"""GPU fp8_row_quant vs the CPU oracle: E4M3 bytes, row scales and group sums must be
bit-identical, the GEMM's group-sum operand must be the documented bf16 hi/lo split of
the oracle's group sums, bit for bit, and the optional fp16 copy must hold exactly the E4M3
values (binary16 bits of the oracle's decoded codes)."""
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
    x16 = torch.full((M, K), float("nan"), dtype=torch.float16, device=cuda())
    w4.fp8_row_quant(Xd, M, K, group if group else 32, X8, s, G, gop, x16=x16)
    torch.cuda.synchronize()
    op = gop.view(torch.int16).cpu().numpy().view(np.uint16) if gop is not None else None
    return np_of(X8), np_of(s), (np_of(G) if G is not None else None), op, x16.view(torch.int16).cpu().numpy().view(np.uint16)


def f16_bits_of_codes(X8):
    return oracle.e4m3_decode(X8).astype(np.float16).view(np.uint16)


def check(X, group, rows=None, op_only=False):
    gX8, gs, gG, gop, gx16 = gpu_row_quant(X, group, op_only)
    bits = synth.bf16_bits(X)
    if rows is not None:
        bits = bits[rows]
        gX8, gs, gx16 = gX8[rows], gs[rows], gx16[rows]
        gG = gG[rows] if gG is not None else None
        gop = gop[rows] if gop is not None else None
    X8, s, G = oracle.row_quant(bits, group)
    assert np.array_equal(gs.view(np.uint32), s.view(np.uint32))
    bad = np.argwhere(gX8 != X8)
    assert bad.size == 0, f"{len(bad)} byte mismatches, first {bad[:3].tolist()}"
    assert np.array_equal(gx16, f16_bits_of_codes(X8))
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
    for g in (32, 64, 128, 256):
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


def rows_below_max(amax_bits, K):
    """Rows of length K that hold every finite bf16 value of magnitude <= the bf16 amax_bits
    (in the first row, amax itself first so that every row's maximum is amax); the rest of
    the last row is zero."""
    pats = np.arange(65536, dtype=np.uint32)
    keep = (pats & 0x7FFF) <= amax_bits
    vals = (pats[keep] << 16).view(np.float32)
    vals = np.concatenate([[np.float32((np.uint32(amax_bits) << 16).view(np.float32))], vals])
    per = K - 1  # each row also carries amax in its first column
    rows = []
    for i in range(0, vals.size, per):
        chunk = vals[i:i + per]
        row = np.zeros(K, np.float32)
        row[0] = vals[0]
        row[1:1 + chunk.size] = chunk
        rows.append(row)
    return rows


@pytest.mark.parametrize("K", [4096, 16384, 32768])
def test_every_value_under_many_row_maxima(K):
    """The kernel divides by the row scale through the row's reciprocal and one exact
    correction step; the codes must equal those of the oracle's IEEE division for every
    bf16 value under row maxima spread over the whole exponent range (K = 4096 takes the
    register-resident warp kernel, K = 16384 the register-resident block kernel, K = 32768
    the three-pass one)."""
    maxima = [0x0001, 0x0080, 0x0A3C, 0x2F11, 0x3300, 0x3C00, 0x3F80, 0x3FFF, 0x4120, 0x43E0,
              0x447F, 0x4B01, 0x5F7F, 0x7A00, 0x7F7F]
    rows = []
    for a in maxima:
        rows += rows_below_max(a, K)
    X = torch.from_numpy(np.array(rows, np.float32)).to(torch.bfloat16)
    check(X, 128)


@pytest.mark.parametrize("K", [512, 3840])
def test_rows_with_infinities(K):
    """A row whose maximum is infinite has an infinite scale: finite values give zero codes
    through the division fallback (the infinite entries themselves are NaN codes and are not
    compared, since the sign of a NaN quotient is not fixed). K = 512 and 3840 take the
    warp-per-row kernel with 4 and 16 chunks per lane."""
    row = np.linspace(-3, 3, K).astype(np.float32)
    row[7] = np.inf
    row2 = row.copy()
    row2[7] = -np.inf
    X = torch.from_numpy(np.array([row, row2])).to(torch.bfloat16)
    gX8, gs, _, _, _ = gpu_row_quant(X, 32)
    X8, s, _ = oracle.row_quant(synth.bf16_bits(X), 32)
    assert np.array_equal(gs.view(np.uint32), s.view(np.uint32))
    finite = np.ones(K, bool)
    finite[7] = False
    assert np.array_equal(gX8[:, finite], X8[:, finite])


def test_fp16_copy_without_codes():
    """Only the fp16 copy (the operand of the groups-32/256 GEMM path): the same values."""
    M, K = 77, 2880
    X = synth.outlier_activation(M, K, 4, 20.0, 2, 11)
    s = torch.empty(M, dtype=torch.float32, device=cuda())
    x16 = torch.full((M, K), float("nan"), dtype=torch.float16, device=cuda())
    w4.fp8_row_quant(X.to(cuda()), M, K, 32, None, s, x16=x16)
    X8, rs, _ = oracle.row_quant(synth.bf16_bits(X), 0)
    torch.cuda.synchronize()
    assert np.array_equal(np_of(s).view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(x16.view(torch.int16).cpu().numpy().view(np.uint16), f16_bits_of_codes(X8))
