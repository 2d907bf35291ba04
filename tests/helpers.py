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
