"""The mixture-of-experts layer around the grouped W4A8 GEMM, each step against the oracle:
the router (exact experts and grouped layout; gates to fp32 rounding), the gathered row
quant (bit-exact), SwiGLU with the row quant of its result (codes decided from fp32 h on
both sides: equal except where the two fp32 evaluations of h straddle an E4M3 rounding
boundary, and every code a correct rounding of the oracle's h within that tolerance), the
combine (bf16 output against the fp64 result rounded to bf16), and the whole layer on a
small configuration and on sampled tokens of the 32-expert one."""
import numpy as np
import pytest
import torch

import oracle
from bit_gemm_wise_b200 import synth, w4
from helpers import bf16_round, cuda, rel_frob, to_dev

pytestmark = pytest.mark.gpu


def logits_of(T, E, seed):
    g = torch.Generator().manual_seed(seed)
    lg = torch.rand(T, E, generator=g)
    if T > 3 and E >= 4:
        lg[3, :4] = lg[3].max() + 0.25  # a four-way tie at the top
    return lg.numpy().astype(np.float32)


def gpu_route(lg, k):
    T, E = lg.shape
    dev = cuda()
    ex = torch.empty(T, k, dtype=torch.int32, device=dev)
    gt = torch.empty(T, k, dtype=torch.float32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    tor = torch.empty(T * k, dtype=torch.int32, device=dev)
    row_of = torch.empty(T, k, dtype=torch.int32, device=dev)
    ws = w4.alloc_moe_route_workspace(T, E, device=dev)
    w4.w4_moe_route(to_dev(lg), T, E, k, ex, gt, off, tor, row_of, ws)
    return ex, gt, off, tor, row_of


@pytest.mark.parametrize("T,E,k", [(4096, 32, 4), (100, 8, 2), (33, 5, 5), (1, 1, 1), (65, 1024, 8),
                                   (300, 100, 3)])
def test_route(T, E, k):
    lg = logits_of(T, E, T + E)
    ex, gt, off, tor, row_of = gpu_route(lg, k)
    rex, rg = oracle.moe_route(lg, k)
    rtor, roff, rrow = oracle.moe_grouping(rex, E)
    torch.cuda.synchronize()
    assert np.array_equal(ex.cpu().numpy(), rex)
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(tor.cpu().numpy(), rtor)
    assert np.array_equal(row_of.cpu().numpy(), rrow)
    assert np.allclose(gt.cpu().numpy(), rg, rtol=2e-6, atol=1e-7)


def test_route_with_nan_and_infinite_logits():
    """Non-finite logits follow the oracle's scan in expert order: a NaN is taken only when it
    is the first expert still untaken; -inf and +inf order like any value."""
    T, E, k = 40, 37, 4
    lg = logits_of(T, E, 9)
    lg[0, 0] = np.nan                  # first expert NaN: chosen first
    lg[1, 5] = np.nan                  # NaN elsewhere: never chosen while finite ones remain
    lg[2, :] = np.nan                  # all NaN: experts 0, 1, 2, 3
    lg[7, 3] = np.nan                  # a NaN after finite ones: skipped
    lg[3, 7] = np.inf
    lg[4, :] = -np.inf                 # all equal: ascending experts
    lg[5, :E - 3] = np.nan             # the first untaken expert is NaN in every round: 0, 1, 2, 3
    lg[6, 1::2] = 0.5                  # many ties
    ex, gt, off, tor, row_of = gpu_route(lg, k)
    rex, rg = oracle.moe_route(lg, k)
    rtor, roff, rrow = oracle.moe_grouping(rex, E)
    torch.cuda.synchronize()
    assert np.array_equal(ex.cpu().numpy(), rex)
    assert np.array_equal(tor.cpu().numpy(), rtor)
    assert np.array_equal(row_of.cpu().numpy(), rrow)
    fin = np.isfinite(rg).all(axis=1)
    assert np.allclose(gt.cpu().numpy()[fin], rg[fin], rtol=2e-6, atol=1e-7)
    assert np.array_equal(np.isnan(gt.cpu().numpy()), np.isnan(rg))


def test_route_rejects_a_short_workspace():
    dev = cuda()
    T, E, k = 64, 32, 2
    lg = torch.zeros(T, E, dtype=torch.float32, device=dev)
    outs = [torch.empty(n, dtype=torch.int32, device=dev) for n in (T * k, T * k, E + 1, T * k, T * k)]
    ws = torch.empty(w4.w4_moe_route_workspace_bytes(T, E) - 4, dtype=torch.uint8, device=dev)
    with pytest.raises(w4.W4Error) as e:
        w4.w4_moe_route(lg, T, E, k, *outs, ws)
    assert e.value.code == 10


def test_gather_row_quant_is_row_quant_of_the_gathered_rows():
    T, K, E, k = 512, 2880, 16, 4
    X = synth.moe_activation()[:T]
    _, _, _, tor, _ = gpu_route(logits_of(T, E, 1), k)
    R = T * k
    X8 = torch.empty(R, K, dtype=torch.uint8, device=cuda())
    sa = torch.empty(R, dtype=torch.float32, device=cuda())
    G = torch.empty(R, K // 32, dtype=torch.float32, device=cuda())
    w4.fp8_row_quant_gather(X.to(cuda()), T, K, 32, tor, R, X8, sa, G)
    rX8, rsa, rG = oracle.row_quant(synth.bf16_bits(X)[tor.cpu().numpy()], 32)
    torch.cuda.synchronize()
    assert np.array_equal(X8.cpu().numpy(), rX8)
    assert np.array_equal(sa.cpu().numpy(), rsa)
    assert np.array_equal(G.cpu().numpy(), rG)


def check_swiglu_codes(X8, sa, Y_bits, H):
    """Codes decided from fp32 h: equal to the oracle's except where h / s lies within a few
    fp32 roundings of a boundary between two E4M3 codes; every GPU code must round the
    oracle's h / s (with the GPU's scale) to within that tolerance."""
    rX8, rsa, rh = oracle.swiglu_row_quant(Y_bits, H)
    assert np.allclose(sa, rsa, rtol=4 * 2.0 ** -23, atol=0)
    same = X8 == rX8
    assert same.mean() > 0.999, same.mean()
    dec = oracle.e4m3_decode(X8).astype(np.float64)
    q = rh.astype(np.float64) / sa.astype(np.float64)[:, None]
    # the E4M3 grid step at |q| (subnormal step 2^-9, else 2^(e-3)), and the rounding error
    e = np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -6)))
    step = np.where(np.abs(q) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (e - 3))
    err = np.abs(dec - np.clip(q, -448, 448))
    assert np.all(err <= 0.5 * step * (1 + 1e-5) + 1e-6 * np.abs(q)), err.max()


@pytest.mark.parametrize("R,H", [(300, 2880), (7, 64), (64, 5760)])
def test_swiglu_quant(R, H):
    g = torch.Generator().manual_seed(R + H)
    Y = (torch.randn(R, 2 * H, generator=g) * 2.0).to(torch.bfloat16)
    Y[0, :H] = 0.0                 # gate 0: h = 0
    Y[1, :8] = torch.tensor([80.0, -80.0, 30.0, -30.0, 1e-3, -1e-3, 3.0, -3.0])
    X8 = torch.empty(R, H, dtype=torch.uint8, device=cuda())
    sa = torch.empty(R, dtype=torch.float32, device=cuda())
    w4.w4_moe_swiglu_quant(Y.to(cuda()), R, H, 32, X8, sa)
    torch.cuda.synchronize()
    check_swiglu_codes(X8.cpu().numpy(), sa.cpu().numpy(), synth.bf16_bits(Y), H)


def test_combine():
    T, k, N = 300, 4, 2880
    rng = np.random.default_rng(5)
    R = T * k
    rows = torch.from_numpy(rng.normal(0, 1, (R, N)).astype(np.float32)).to(torch.bfloat16)
    row_of = rng.permutation(R).reshape(T, k).astype(np.int32)
    gates = rng.random((T, k)).astype(np.float32)
    gates /= gates.sum(1, keepdims=True)
    y = torch.empty(T, N, dtype=torch.bfloat16, device=cuda())
    w4.w4_moe_combine(rows.to(cuda()), N, R, to_dev(row_of), to_dev(gates), T, k, y)
    ref = oracle.moe_combine(rows.double().numpy(), row_of, gates.astype(np.float64))
    torch.cuda.synchronize()
    assert rel_frob(bf16_round(ref), y.double().cpu().numpy()) <= 1e-3


def quantized_experts(E, N, K, g, base, seed=0):
    out = [oracle.quantize(synth.bf16_bits(synth.normal((N, K), 0.02, seed, base + e)), g, "asym", [1.0], False)[:3]
           for e in range(E)]
    return tuple(np.stack([o[i] for o in out]) for i in range(3))


def upload_experts(q, N, K, g):
    E = q[0].shape[0]
    nb = w4.w4_prepack_bytes(N, K, g, w4.W4_LAYOUT_GEMM)
    packed = torch.empty(E * nb, dtype=torch.uint8, device=cuda())
    for e in range(E):
        w4.w4_prepack(to_dev(q[0][e]), to_dev(q[1][e].view(np.int16)), to_dev(q[2][e]), N, K, g, "asym",
                      w4.W4_LAYOUT_GEMM, packed[e * nb:])
    return packed


def moe_layer_gpu(X, lg, k, pgu, pdn, H, K, g):
    """The layer through the C ABI: route, gathered row quant, gate_up GEMM, SwiGLU + row
    quant, down GEMM, combine."""
    T, E = lg.shape
    dev = cuda()
    ex, gt, off, tor, row_of = gpu_route(lg, k)
    R = T * k
    # group 32: the GEMMs take the fp16 copy of the E4M3 activations, so the dispatch writes
    # only that copy; the SwiGLU quant writes both (the codes are checked below)
    X16 = torch.empty(R, K, dtype=torch.float16, device=dev)
    sa = torch.empty(R, dtype=torch.float32, device=dev)
    w4.fp8_row_quant_gather(X, T, K, g, tor, R, None, sa, x16=X16)
    Ygu = torch.empty(R, 2 * H, dtype=torch.bfloat16, device=dev)
    w4.w4a8_grouped_gemm(None, sa, None, off, E, R, pgu, 2 * H, K, g, "asym", Ygu, X16=X16)
    H8 = torch.empty(R, H, dtype=torch.uint8, device=dev)
    H16 = torch.empty(R, H, dtype=torch.float16, device=dev)
    sh = torch.empty(R, dtype=torch.float32, device=dev)
    w4.w4_moe_swiglu_quant(Ygu, R, H, g, H8, sh, x16=H16)
    Yd = torch.empty(R, K, dtype=torch.bfloat16, device=dev)
    w4.w4a8_grouped_gemm(None, sh, None, off, E, R, pdn, K, H, g, "asym", Yd, X16=H16)
    y = torch.empty(T, K, dtype=torch.bfloat16, device=dev)
    w4.w4_moe_combine(Yd, K, R, row_of, gt, T, k, y)
    return y, dict(Ygu=Ygu, H8=H8, sh=sh, Yd=Yd)


def test_layer_small():
    E, k, T, K, H, g = 8, 2, 64, 256, 128, 32
    X = synth.normal((T, K), 1.0, 3, 1)
    lg = logits_of(T, E, 7)
    gu = quantized_experts(E, 2 * H, K, g, 300)
    dn = quantized_experts(E, K, H, g, 400)
    y, mid = moe_layer_gpu(X.to(cuda()), lg, k, upload_experts(gu, 2 * H, K, g), upload_experts(dn, K, H, g), H, K, g)
    ref, rmid = oracle.moe_layer_ref(synth.bf16_bits(X), lg, k, gu, dn, g, "asym")
    torch.cuda.synchronize()
    # the intermediate the two sides quantize is bf16 on both; a handful of its elements may
    # round differently (fp32 vs fp64 products), so codes may differ at rounding boundaries
    check_swiglu_codes(mid["H8"].cpu().numpy(), mid["sh"].cpu().numpy(),
                       synth.bf16_bits(mid["Ygu"].cpu()), H)
    e = rel_frob(ref, y.double().cpu().numpy())
    assert e <= 2e-2 and e <= 5e-3, e


def test_layer_32_experts_sampled_tokens():
    """The 32-expert, top-4 layer at full size (4096 tokens, 2880 -> 5760 -> 2880, group 32),
    16 sampled tokens against the oracle's layer."""
    c = synth.MOE
    E, k, T, K, H, g = c["E"], c["top_k"], c["tokens"], c["K"], c["N_down"], c["group"]
    X = synth.moe_activation()
    gl = torch.Generator().manual_seed(60)
    lg = torch.rand(T, E, generator=gl).numpy().astype(np.float32)
    qgu = [oracle.quantize(synth.bf16_bits(synth.moe_weight("gate_up", e)), g, "asym", [1.0], False)[:3]
           for e in range(E)]
    qdn = [oracle.quantize(synth.bf16_bits(synth.moe_weight("down", e)), g, "asym", [1.0], False)[:3]
           for e in range(E)]
    gu = tuple(np.stack([o[i] for o in qgu]) for i in range(3))
    dn = tuple(np.stack([o[i] for o in qdn]) for i in range(3))
    y, _ = moe_layer_gpu(X.to(cuda()), lg, k, upload_experts(gu, 2 * H, K, g), upload_experts(dn, K, H, g), H, K, g)
    toks = np.linspace(0, T - 1, 16).astype(int)
    ref, _ = oracle.moe_layer_ref(synth.bf16_bits(X), lg, k, gu, dn, g, "asym", tokens=toks)
    torch.cuda.synchronize()
    e = rel_frob(ref[toks], y.double().cpu().numpy()[toks])
    assert e <= 2e-2 and e <= 5e-3, e
    assert w4.w4_device_status() == 0
