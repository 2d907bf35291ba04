"""GPU w4_quantize vs the CPU oracle: codes, scales, zeros and chosen ratio must be
bit-identical (integer work decided by fp32 arithmetic in the same order on both sides)."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import cuda, np_of, np_u16, to_dev

pytestmark = pytest.mark.gpu


def gpu_quantize(Wb, group, mode, grid):
    N, K = Wb.shape
    codes, scales, zeros, chosen = w4.alloc_quantized(N, K, group, mode)
    w4.w4_quantize(Wb, N, K, group, mode, grid, codes, scales, zeros, chosen)
    torch.cuda.synchronize()
    return (np_of(codes), np_u16(scales), None if zeros is None else np_of(zeros), np_of(chosen))


def assert_same(gpu, ref, rows=None):
    names = ("codes", "scales", "zeros", "chosen")
    for name, g, r in zip(names, gpu, ref):
        if r is None:
            assert g is None
            continue
        gg = g if rows is None else g[rows]
        assert gg.shape == r.shape, name
        bad = np.argwhere(gg != r)
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first at {bad[:3].tolist()}"


def check(W_bf16, group, mode, grid, rows=None):
    Wd = W_bf16.to(cuda())
    gpu = gpu_quantize(Wd, group, mode, grid)
    bits = synth.bf16_bits(W_bf16)
    if rows is not None:
        bits = bits[rows]
    ref = oracle.quantize(bits, group, mode, grid)
    assert_same(gpu, ref, rows)
    return gpu


def test_single_layer_sym_g32():
    W, _ = synth.single_layer()
    check(W, 32, "sym", [1.0])


def test_single_layer_page_orientation():
    W, _ = synth.single_layer_page_orientation()
    check(W, 32, "sym", [1.0])


@pytest.mark.parametrize("K,N", synth.DECODE_SHAPES)
def test_decode_shapes_full_size_sampled_rows(K, N):
    """Full-size 8B decode weights, asym g128, 20-ratio clip search; the GPU quantizes the
    whole matrix, the oracle 192 rows spread over it (rows are independent)."""
    W = synth.decode_weight(K, N)
    rows = np.unique(np.concatenate([np.arange(64), np.linspace(0, N - 1, 96).astype(int), np.arange(N - 32, N)]))
    check(W, 128, "asym", synth.clip_grid_20(), rows)


def test_decode_small_full_compare():
    W = synth.decode_weight(4096, 1024)
    check(W, 128, "asym", synth.clip_grid_20())


@pytest.mark.parametrize("group", [32, 64, 128, 256])
@pytest.mark.parametrize("mode", ["sym", "asym"])
@pytest.mark.parametrize("grid", ["one", "page", "twenty"])
def test_groups_modes_grids(group, mode, grid):
    g = {"one": [1.0], "page": synth.clip_grid_page(), "twenty": synth.clip_grid_20()}[grid]
    K = 384 if group < 256 else 768                         # 3 groups of 128, 3 of 256
    W = synth.student_t3_weight(77, K, 0, 900 + group)     # ragged N, heavy tails
    check(W, group, mode, g)


def test_8b_weight_set_slice():
    """A layer of the Student-t(3) 8B set (gate projection): rows sampled."""
    W = synth.llama8b_weight(0, "gate")
    rows = np.linspace(0, W.shape[0] - 1, 128).astype(int)
    check(W, 128, "asym", synth.clip_grid_20(), rows)


def test_moe_expert_weights_g32():
    W = synth.moe_weight("gate_up", 3)
    rows = np.linspace(0, W.shape[0] - 1, 256).astype(int)
    check(W, 32, "asym", [1.0], rows)


def _edge_matrix(K=128):
    rng = np.random.default_rng(5)
    rows = []
    rows.append(np.zeros(K))                                   # all zero -> s = 1 guard
    rows.append(np.full(K, 0.37))                              # constant positive
    rows.append(np.full(K, -2.5))                              # constant negative
    rows.append(1.0 + rng.uniform(0, 0.01, K))                 # one-signed, tight: zero far below 0
    rows.append(-50.0 - rng.uniform(0, 0.5, K))                # one-signed negative
    rows.append(rng.normal(0, 1e-6, K))                        # tiny: fp16 subnormal scales
    rows.append(rng.normal(0, 1e-9, K))                        # tinier: scale rounds to 0 -> 1
    r = rng.normal(0, 0.02, K); r[7] = 40.0; rows.append(r)    # one far outlier
    r = rng.normal(0, 1.0, K) * 3e4; rows.append(r)            # large: fp16 scale near its max
    r = (np.arange(K) % 15 - 7) * 0.125; rows.append(r)        # exact lattice, ties
    r = np.linspace(-0.3125, 1.5625, K); rows.append(r)        # zero point tie 2.5
    r = rng.choice([-1.0, 1.0], K) * 0.5; rows.append(r)       # two values
    return torch.tensor(np.array(rows), dtype=torch.float32).to(torch.bfloat16)


@pytest.mark.parametrize("mode", ["sym", "asym"])
@pytest.mark.parametrize("group", [32, 128, 256])
def test_edge_blocks(mode, group):
    check(_edge_matrix(max(128, group)), group, mode, synth.clip_grid_20())


def test_tiny_shapes():
    for N, K, g in [(1, 32, 32), (1, 64, 64), (3, 128, 128), (5, 96, 32), (2, 4096, 128)]:
        W = synth.normal((N, K), 0.02, 1, N * 7 + K)
        check(W, g, "asym", synth.clip_grid_20())
        check(W, g, "sym", [1.0, 0.9])


def test_deterministic_repeat():
    W = synth.decode_weight(4096, 1024).to(cuda())
    a = gpu_quantize(W, 128, "asym", synth.clip_grid_20())
    b = gpu_quantize(W, 128, "asym", synth.clip_grid_20())
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_no_device_status_after_runs():
    assert w4.w4_device_status() == 0
