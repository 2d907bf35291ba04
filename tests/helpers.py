"""Shared helpers of the tests (no method arithmetic): device selection, conversions
between torch tensors and the numpy arrays the oracle takes."""
import numpy as np
import torch

from bit_gemm_wise_b200 import synth


def cuda():
    return torch.device("cuda:0")


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(cuda())


def np_u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def np_of(t):
    return t.detach().cpu().contiguous().numpy()


def bf16_dev(t):
    return t.to(torch.bfloat16).contiguous().to(cuda())


def rel_frob(ref, got):
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    return float(np.linalg.norm(ref - got) / max(np.linalg.norm(ref), 1e-300))


def bf16_round(a):
    """Round fp64 values to bf16 (RNE) through torch's cast, returned as fp64."""
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.float32).to(torch.bfloat16).double().numpy()


bf16_bits = synth.bf16_bits


def gsum_operand(G, K, group):
    """The W4A8 GEMM's group-sum operand (the format w4.h documents for fp8_row_quant's
    gsum_op) built from fp32 group sums G [M, J]: row m = [hi | lo | hi | 0 ...] with
    hi = bf16(G) and lo = bf16(G - hi), both round-to-nearest-even, padded to a multiple of
    32 columns. Returned as uint16 bit patterns."""
    G = np.asarray(G, np.float32)
    M, J = G.shape
    assert J == K // group
    cols = (3 * J + 31) // 32 * 32
    hi = torch.from_numpy(G).to(torch.bfloat16)
    lo = (torch.from_numpy(G) - hi.float()).to(torch.bfloat16)
    h = hi.view(torch.int16).numpy().view(np.uint16)
    l = lo.view(torch.int16).numpy().view(np.uint16)
    out = np.zeros((M, cols), np.uint16)
    out[:, :J], out[:, J:2 * J], out[:, 2 * J:3 * J] = h, l, h
    return out
