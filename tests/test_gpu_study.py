"""The group-size / clip-grid study measured on the built path: for every layer, mode, group
size (32, 64, 128, 256) and clip grid of the CPU study (test_study_group_clip.py), the GPU
quantizer's codes, scales and zeros must equal the oracle's bit for bit, and the output error
of the GPU W4A16 GEMV (16 activation rows, fp32 output) against the unquantized product must
equal the oracle's to within the GEMV's own rounding (1e-5 absolute on a relative error).
Run with -s to print the table as measured on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import cuda, np_u16, to_dev
from test_study_group_clip import GRIDS, GROUPS, layers

pytestmark = pytest.mark.gpu


def test_study_on_gpu():
    print()
    print(f"{'layer':46s} {'mode':5s} {'g':>4s} {'grid':14s} {'GPU output err':>14s} {'oracle':>9s}")
    for name, W, X in layers():
        N, K = W.shape
        M = X.shape[0]
        bits = synth.bf16_bits(W)
        w = W.float().numpy().astype(np.float64)
        x = X.float().numpy().astype(np.float64)
        y = x @ w.T
        Wd, Xd = W.to(cuda()), X.to(cuda())
        for mode in ("sym", "asym"):
            for g in GROUPS:
                for gname, grid in GRIDS.items():
                    codes, scales, zeros, _ = w4.alloc_quantized(N, K, g, mode, chosen=False)
                    w4.w4_quantize(Wd, N, K, g, mode, grid, codes, scales, zeros, None)
                    rc, rs, rz, _ = oracle.quantize(bits, g, mode, grid, want_chosen=False)
                    packed = w4.alloc_packed(N, K, g, w4.W4_LAYOUT_GEMV)
                    w4.w4_prepack(codes, scales, zeros, N, K, g, mode, w4.W4_LAYOUT_GEMV, packed)
                    out = torch.empty(M, N, dtype=torch.float32, device=cuda())
                    w4.w4a16_gemv(Xd, M, packed, N, K, g, mode, out, w4.W4_OUT_FP32,
                                  w4.alloc_gemv_workspace(N, K, g))
                    torch.cuda.synchronize()
                    assert np.array_equal(codes.cpu().numpy(), rc)
                    assert np.array_equal(np_u16(scales), rs)
                    if mode == "asym":
                        assert np.array_equal(zeros.cpu().numpy(), rz)
                    wd = oracle.dequantize(rc, rs, rz, g, mode)
                    ref_err = oracle.rel_error(y, x @ wd.T)
                    gpu_err = oracle.rel_error(y, out.cpu().numpy().astype(np.float64))
                    print(f"{name:46s} {mode:5s} {g:4d} {gname:14s} {100 * gpu_err:13.4f}% {100 * ref_err:8.4f}%")
                    assert abs(gpu_err - ref_err) <= 1e-5, (name, mode, g, gname, gpu_err, ref_err)
