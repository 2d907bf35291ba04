"""The allocation-free GEMV entry point (w4a16_gemv_noalloc) against the regular one.

Some callers cannot allocate device memory on their hot path -- a plug-in inside another
runtime that owns all device memory, or a decode loop that cannot afford cudaMalloc's
implicit device synchronisation -- so w4a16_gemv_noalloc keeps its scratch in a fixed array
inside the library instead of a caller-provided workspace. It must give the same outputs as
w4a16_gemv with a workspace, call after call (the shared array keeps the previous call's
contents, so a second call in a row is part of the check). The scratch holds the partial sums
of rows split along K over several blocks (rows too long for one block), so the cases with
K = 65536 are the ones that use it; the others check that the entry point is also right when
no scratch is needed. This file is collected last so that a failure here never hides the
other tests' results, and it builds its own inputs.
"""
import numpy as np
import pytest
import torch

from bit_gemm_wise_b200 import synth, w4

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4   # the tolerance of the fp32-output GEMV tests
TOL_BF16 = 1e-3  # the tolerance of the bf16-output GEMV tests


def rel(a, b):
    a = a.double()
    b = b.double()
    return float((a - b).norm() / b.norm().clamp_min(1e-300))


def packed_weight(N, K, g, seed):
    dev = torch.device("cuda:0")
    W = synth.normal((N, K), 0.02, seed, 7).to(dev)
    codes, scales, zeros, _ = w4.alloc_quantized(N, K, g, "asym", device=dev, chosen=False)
    w4.w4_quantize(W, N, K, g, "asym", synth.clip_grid_20(), codes, scales, zeros, None)
    p = w4.alloc_packed(N, K, g, w4.W4_LAYOUT_GEMV, device=dev)
    w4.w4_prepack(codes, scales, zeros, N, K, g, "asym", w4.W4_LAYOUT_GEMV, p)
    return p


# (N, K, M): decode shapes (whole rows per block, no scratch), rows split along K (the scratch
# holds their partial sums) at one and three activation rows, a ragged shape and the largest M
CASES = [(1024, 4096, 1), (4096, 14336, 1), (300, 65536, 1), (100, 65536, 3), (77, 320, 3), (4096, 4096, 16)]


@pytest.mark.parametrize("N,K,M", CASES)
@pytest.mark.parametrize("flags", [0, w4.W4_OUT_FP32])
def test_noalloc_matches_workspace_entry_point(N, K, M, flags):
    dev = torch.device("cuda:0")
    g = 64 if K % 128 else 128
    p = packed_weight(N, K, g, N + K)
    x = synth.normal((M, K), 1.0, 3, M).to(dev)
    dt = torch.float32 if flags & w4.W4_OUT_FP32 else torch.bfloat16
    ws = w4.alloc_gemv_workspace(N, K, g, device=dev)
    ref = torch.full((M, N), float("nan"), dtype=dt, device=dev)
    w4.w4a16_gemv(x, M, p, N, K, g, "asym", ref, flags, ws)
    torch.cuda.synchronize()
    assert torch.isfinite(ref).all() and w4.w4_device_status() == 0
    tol = TOL_F32 if dt == torch.float32 else TOL_BF16
    for _ in range(2):  # two calls in a row on the shared scratch
        got = torch.full((M, N), float("nan"), dtype=dt, device=dev)
        w4.w4a16_gemv_noalloc(x, M, p, N, K, g, "asym", got, flags)
        torch.cuda.synchronize()
        assert torch.isfinite(got).all()
        assert rel(got, ref) <= tol
    assert w4.w4_device_status() == 0


def test_noalloc_chain_on_one_stream_with_overlap():
    """Two calls in a row on one stream with W4_OVERLAP_PREVIOUS, both splitting their rows
    along K: each call clears its counters with a memset on the stream, which orders it
    after the previous call; the results must equal the workspace entry point's."""
    dev = torch.device("cuda:0")
    N, K, g = 300, 65536, 128
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert w4.w4a16_gemv_schedule(1, N, K, g, sms)["k_parts"] >= 2
    p = packed_weight(N, K, g, 5)
    xs = [synth.normal((1, K), 1.0, 3, 40 + i).to(dev) for i in range(2)]
    ws = w4.alloc_gemv_workspace(N, K, g, device=dev)
    refs = []
    for x in xs:
        r = torch.empty(1, N, dtype=torch.float32, device=dev)
        w4.w4a16_gemv(x, 1, p, N, K, g, "asym", r, w4.W4_OUT_FP32, ws)
        refs.append(r)
    outs = [torch.full((1, N), float("nan"), dtype=torch.float32, device=dev) for _ in xs]
    for x, o in zip(xs, outs):
        w4.w4a16_gemv_noalloc(x, 1, p, N, K, g, "asym", o, w4.W4_OUT_FP32 | w4.W4_OVERLAP_PREVIOUS)
    torch.cuda.synchronize()
    for o, r in zip(outs, refs):
        assert torch.isfinite(o).all()
        assert rel(o, r) <= TOL_F32
    assert w4.w4_device_status() == 0


def test_noalloc_rejects_requests_beyond_its_scratch():
    dev = torch.device("cuda:0")
    limit = w4.w4a16_gemv_noalloc_scratch_limit()
    assert limit == 1 << 20
    # rows split along K need kparts * M * N * 4 bytes of partial sums: 2 parts of 200000 rows
    N = 200000
    dummy = torch.zeros(256, dtype=torch.uint8, device=dev)
    x = torch.zeros(1, 65536, dtype=torch.bfloat16, device=dev)
    with pytest.raises(w4.W4Error) as e:
        w4.w4a16_gemv_noalloc(x, 1, dummy, N, 65536, 128, "asym", dummy, 0)
    assert e.value.code == 11
    torch.cuda.synchronize()
