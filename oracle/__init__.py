"""CPU oracle for the W4 quantizer, the FP8 row quantizer and the W4A16 / W4A8 products.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package. The product path (the
``bit_gemm_wise_b200`` package and its CUDA library) never imports, links or runs it.

The arithmetic lives in ``w4_oracle.c`` (plain scalar C, one IEEE fp32 operation per written
operation, fp64 for the reference products). This module only builds it with gcc and moves
numpy arrays in and out. ``rel_error`` and ``bits_per_weight`` restate the closed forms of
"Quantizing LLMs Without Guesswork", "Quantize, then dequantize".

Parity pins: every function is pinned in ``tests/test_oracle_pins.py`` against values the
pages print, closed forms, brute force or an independent library routine.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

SYM, ASYM = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: -O2, no FMA contraction, no fast-math, OpenMP over rows."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-fvisibility=hidden", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        lib.o_bf16_to_f32.restype = ctypes.c_float
        lib.o_bf16_to_f32.argtypes = [ctypes.c_uint16]
        lib.o_f32_to_f16_bits.restype = ctypes.c_uint16
        lib.o_f32_to_f16_bits.argtypes = [ctypes.c_float]
        lib.o_f16_bits_to_f32.restype = ctypes.c_float
        lib.o_f16_bits_to_f32.argtypes = [ctypes.c_uint16]
        lib.o_e4m3_encode.restype = ctypes.c_uint8
        lib.o_e4m3_encode.argtypes = [ctypes.c_float]
        lib.o_e4m3_decode.restype = ctypes.c_float
        lib.o_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.o_quantize.restype = I
        lib.o_quantize.argtypes = [P, I64, I64, I, I, P, I, P, P, P, P]
        lib.o_block_sse.restype = ctypes.c_float
        lib.o_block_sse.argtypes = [P, I, I, ctypes.c_float]
        lib.o_dequantize.restype = None
        lib.o_dequantize.argtypes = [P, P, P, I64, I64, I, I, P]
        lib.o_row_quant.restype = None
        lib.o_row_quant.argtypes = [P, I64, I64, I, P, P, P]
        lib.o_gemv_ref.restype = None
        lib.o_gemv_ref.argtypes = [P, I64, P, P, P, I64, I64, I, I, P]
        lib.o_w4a8_ref_pairs.restype = None
        lib.o_w4a8_ref_pairs.argtypes = [P, P, I64, P, P, P, I64, I, I, P, P, P, I64, P]
        lib.o_fake_quant.restype = None
        lib.o_fake_quant.argtypes = [P, I64, I64, I, I, P, P]
        lib.o_nf4_levels.restype = None
        lib.o_nf4_levels.argtypes = [P]
        lib.o_nf4_quantize.restype = I
        lib.o_nf4_quantize.argtypes = [P, I64, I64, P, P]
        lib.o_nf4_gemv_ref.restype = None
        lib.o_nf4_gemv_ref.argtypes = [P, I64, P, P, I64, I64, P]
        lib.o_moe_route.restype = None
        lib.o_moe_route.argtypes = [P, I64, I, I, P, P]
        lib.o_swiglu_row_quant.restype = None
        lib.o_swiglu_row_quant.argtypes = [P, I64, I64, P, P, P]
        lib.o_moe_combine.restype = None
        lib.o_moe_combine.argtypes = [P, I64, P, P, I64, I, P]
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _mode(mode) -> int:
    if mode in (ASYM, "asym"):
        return ASYM
    if mode in (SYM, "sym"):
        return SYM
    raise ValueError(mode)


# ------------------------------------------------------------------ number formats

def bf16_to_f32(bits) -> np.ndarray:
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_f16_bits(x) -> np.ndarray:
    lib = _load()
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint16)
    flat, of = x.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        of[i] = lib.o_f32_to_f16_bits(float(flat[i]))
    return out


def f16_bits_to_f32(h) -> np.ndarray:
    lib = _load()
    h = _c(h, np.uint16)
    out = np.empty(h.shape, np.float32)
    flat, of = h.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        of[i] = lib.o_f16_bits_to_f32(int(flat[i]))
    return out


def e4m3_encode(x) -> np.ndarray:
    lib = _load()
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    flat, of = x.reshape(-1), out.reshape(-1)
    for i in range(flat.size):
        of[i] = lib.o_e4m3_encode(float(flat[i]))
    return out


def e4m3_decode(b) -> np.ndarray:
    """Vectorised through a 256-entry table built by the oracle's own decoder."""
    lib = _load()
    table = np.array([lib.o_e4m3_decode(i) for i in range(256)], dtype=np.float32)
    return table[_c(b, np.uint8)]


# ------------------------------------------------------------------ quantizer

def quantize(W_bits, group: int, mode, grid, want_chosen: bool = True):
    """W_bits: uint16 bf16 patterns [N, K]. Returns (codes u8 [N,K/2], scales u16 fp16 bits
    [N,K/g], zeros i16 [N,K/g] or None for sym, chosen u8 [N,K/g] or None)."""
    lib = _load()
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    m = _mode(mode)
    grid = _c(grid, np.float32)
    J = K // group
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, J), np.uint16)
    zeros = np.empty((N, J), np.int16) if m == ASYM else None
    chosen = np.empty((N, J), np.uint8) if want_chosen else None
    rc = lib.o_quantize(_p(W), N, K, group, m, _p(grid), grid.size, _p(codes), _p(scales),
                        _p(zeros), _p(chosen))
    if rc:
        raise ValueError("oracle quantize: bad arguments")
    return codes, scales, zeros, chosen


def block_sse(w_bits, mode, r: float) -> float:
    lib = _load()
    w = _c(w_bits, np.uint16)
    return float(lib.o_block_sse(_p(w), w.size, _mode(mode), float(r)))


def dequantize(codes, scales, zeros, group: int, mode) -> np.ndarray:
    lib = _load()
    codes = _c(codes, np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 2
    out = np.empty((N, K), np.float64)
    z = None if zeros is None else _c(zeros, np.int16)
    lib.o_dequantize(_p(codes), _p(_c(scales, np.uint16)), _p(z), N, K, group, _mode(mode), _p(out))
    return out


def unpack_codes(codes) -> np.ndarray:
    codes = _c(codes, np.uint8)
    q = np.empty((codes.shape[0], codes.shape[1] * 2), np.uint8)
    q[:, 0::2] = codes & 0xF
    q[:, 1::2] = codes >> 4
    return q


# ------------------------------------------------------------------ activations

def row_quant(X_bits, group: int = 0):
    """X_bits: uint16 bf16 [M, K]. Returns (X8 u8 [M,K], row_scale f32 [M], gsum f32 [M,K/g]
    or None when group == 0)."""
    lib = _load()
    X = _c(X_bits, np.uint16)
    M, K = X.shape
    X8 = np.empty((M, K), np.uint8)
    s = np.empty(M, np.float32)
    G = np.empty((M, K // group), np.float32) if group else None
    lib.o_row_quant(_p(X), M, K, group, _p(X8), _p(s), _p(G))
    return X8, s, G


# ------------------------------------------------------------------ reference products

def gemv_ref(x_bits, codes, scales, zeros, group: int, mode) -> np.ndarray:
    """fp64 y[M,N] = x @ W'^T with W' the dequantized weight (scalar C loops)."""
    lib = _load()
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = _c(codes, np.uint8)
    N = codes.shape[0]
    y = np.empty((M, N), np.float64)
    z = None if zeros is None else _c(zeros, np.int16)
    lib.o_gemv_ref(_p(x), M, _p(codes), _p(_c(scales, np.uint16)), _p(z), N, K, group,
                   _mode(mode), _p(y))
    return y


def w4a8_ref_pairs(X8, s_a, codes, scales, zeros, group: int, mode, rows, cols,
                   expert_of_row=None) -> np.ndarray:
    """fp64 Y[m,n] for the listed (m, n) pairs: the product of the dequantized FP8
    activations (e4m3 value * row scale) and the dequantized INT4 weights. For grouped
    (per-expert) weights, codes/scales/zeros are stacked [E, N, ...] and expert_of_row gives
    the expert of every activation row."""
    lib = _load()
    X8 = _c(X8, np.uint8)
    K = X8.shape[1]
    codes = _c(codes, np.uint8)
    N = codes.shape[-2]
    rows = _c(rows, np.int64)
    cols = _c(cols, np.int64)
    out = np.empty(rows.size, np.float64)
    z = None if zeros is None else _c(zeros, np.int16)
    e = None if expert_of_row is None else _c(expert_of_row, np.int32)
    lib.o_w4a8_ref_pairs(_p(X8), _p(_c(s_a, np.float32)), K, _p(codes), _p(_c(scales, np.uint16)),
                         _p(z), N, group, _mode(mode), _p(e), _p(rows), _p(cols), rows.size, _p(out))
    return out


def w4a8_ref_dense(X8, s_a, codes, scales, zeros, group: int, mode) -> np.ndarray:
    """fp64 Y = A' @ W'^T for small shapes, with A' = e4m3val(X8) * s_a and W' the dequantized
    weight; the matmul is numpy's fp64 routine."""
    A = e4m3_decode(X8).astype(np.float64) * np.asarray(s_a, np.float64)[:, None]
    W = dequantize(codes, scales, zeros, group, mode)
    return A @ W.T


# ------------------------------------------------------------------ NF4 comparator

def nf4_levels() -> np.ndarray:
    """The 16 NF4 levels (fp32, ascending)."""
    lib = _load()
    out = np.empty(16, np.float32)
    lib.o_nf4_levels(_p(out))
    return out


def nf4_quantize(W_bits):
    """NF4 in blocks of 64: (codes u8 [N, K/2] packed as the INT4 codes, absmax f32 [N, K/64])."""
    lib = _load()
    W = _c(W_bits, np.uint16)
    N, K = W.shape
    codes = np.empty((N, K // 2), np.uint8)
    absmax = np.empty((N, K // 64), np.float32)
    if lib.o_nf4_quantize(_p(W), N, K, _p(codes), _p(absmax)):
        raise ValueError("oracle nf4_quantize: K must be a multiple of 64")
    return codes, absmax


def nf4_gemv_ref(x_bits, codes, absmax) -> np.ndarray:
    lib = _load()
    x = _c(x_bits, np.uint16)
    M, K = x.shape
    codes = _c(codes, np.uint8)
    N = codes.shape[0]
    y = np.empty((M, N), np.float64)
    lib.o_nf4_gemv_ref(_p(x), M, _p(codes), _p(_c(absmax, np.float32)), N, K, _p(y))
    return y


# ------------------------------------------------------------------ mixture-of-experts layer

def moe_route(logits, k: int):
    """Top-k experts per token (descending logit, equal logits in ascending expert order) and
    their gate weights, the fp64 softmax of the k selected logits. logits: fp32 [T, E]."""
    lib = _load()
    lg = _c(logits, np.float32)
    T, E = lg.shape
    experts = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float64)
    lib.o_moe_route(_p(lg), T, E, k, _p(experts), _p(gates))
    return experts, gates


def moe_grouping(experts, E: int):
    """Rows of the expert-grouped layout: for each expert, its tokens in ascending order.
    Returns (token_of_row int64 [T*k], expert_row_offsets int32 [E+1], row_of int32 [T, k])
    with row_of[t, i] the grouped row holding token t's i-th expert."""
    experts = np.asarray(experts, np.int64)
    T, k = experts.shape
    off = np.zeros(E + 1, np.int32)
    token_of_row = []
    row_of = np.empty((T, k), np.int32)
    for e in range(E):
        toks = [t for t in range(T) for i in range(k) if experts[t, i] == e]
        for t in toks:
            i = int(np.nonzero(experts[t] == e)[0][0])
            row_of[t, i] = len(token_of_row)
            token_of_row.append(t)
        off[e + 1] = len(token_of_row)
    return np.asarray(token_of_row, np.int64), off, row_of


def swiglu_row_quant(Y_bits, H: int):
    """SwiGLU of the gate_up output (bf16 [R, 2H]: gate | up) and the per-row E4M3 quant of
    the result. Returns (X8 u8 [R, H], row_scale f32 [R], h f32 [R, H])."""
    lib = _load()
    Y = _c(Y_bits, np.uint16)
    R = Y.shape[0]
    assert Y.shape[1] == 2 * H
    X8 = np.empty((R, H), np.uint8)
    s = np.empty(R, np.float32)
    h = np.empty((R, H), np.float32)
    lib.o_swiglu_row_quant(_p(Y), R, H, _p(X8), _p(s), _p(h))
    return X8, s, h


def moe_combine(rows, row_of, gates) -> np.ndarray:
    """y[t] = sum_i gates[t, i] * rows[row_of[t, i]] in fp64."""
    lib = _load()
    rows = _c(rows, np.float64)
    row_of = _c(row_of, np.int32)
    gates = _c(gates, np.float64)
    T, k = row_of.shape
    N = rows.shape[1]
    y = np.empty((T, N), np.float64)
    lib.o_moe_combine(_p(rows), N, _p(row_of), _p(gates), T, k, _p(y))
    return y


def moe_layer_ref(X_bits, logits, k: int, gu, dn, group: int, mode, tokens=None):
    """The whole expert layer in the oracle's arithmetic: route; per-row E4M3 quant of every
    routed token row; fp64 W4A8 gate_up product rounded to bf16 (the GEMM's output type);
    SwiGLU and the per-row E4M3 quant of its result; fp64 W4A8 down product; weighted
    combine. gu / dn: (codes, scales, zeros) stacked over experts [E, N, ...]. tokens (optional):
    evaluate only these tokens (the routing is still computed for all of them; rows of other
    tokens are left zero and their outputs are not meaningful). Dense fp64 matmuls over an
    expert's rows. Returns (y fp64 [T, N_down], intermediates dict)."""
    import torch
    experts, gates = moe_route(logits, k)
    E = gu[0].shape[0]
    token_of_row, off, row_of = moe_grouping(experts, E)
    Xr = np.asarray(X_bits, np.uint16)[token_of_row]
    keep = np.ones(token_of_row.size, bool) if tokens is None else np.isin(token_of_row, np.asarray(tokens))
    X8, s_a, _ = row_quant(Xr, 0)
    A = e4m3_decode(X8).astype(np.float64) * s_a.astype(np.float64)[:, None]
    H = gu[0].shape[1] // 2
    Ygu = np.zeros((Xr.shape[0], 2 * H), np.float64)
    for e in range(E):
        sel = np.arange(off[e], off[e + 1])[keep[off[e]:off[e + 1]]]
        if sel.size:
            Ygu[sel] = A[sel] @ dequantize(gu[0][e], gu[1][e], None if gu[2] is None else gu[2][e], group, mode).T
    Ygu_bits = torch.from_numpy(Ygu).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    H8, s_h, _ = swiglu_row_quant(Ygu_bits, H)
    Ah = e4m3_decode(H8).astype(np.float64) * s_h.astype(np.float64)[:, None]
    Nd = dn[0].shape[1]
    Yd = np.zeros((Xr.shape[0], Nd), np.float64)
    for e in range(E):
        sel = np.arange(off[e], off[e + 1])[keep[off[e]:off[e + 1]]]
        if sel.size:
            Yd[sel] = Ah[sel] @ dequantize(dn[0][e], dn[1][e], None if dn[2] is None else dn[2][e], group, mode).T
    y = moe_combine(Yd, row_of, gates)
    return y, dict(experts=experts, gates=gates, token_of_row=token_of_row, offsets=off, row_of=row_of,
                   X8=X8, s_a=s_a, gate_up_bits=Ygu_bits, H8=H8, s_h=s_h, down=Yd)


# ------------------------------------------------------------------ page formulas

def fake_quant(x, bits: int, symmetric: bool, block) -> tuple[np.ndarray, np.ndarray]:
    """Generic b-bit fake quantization of a float64 array in blocks of ``block`` consecutive
    values (``block=None``: one block for the whole array, per-tensor)."""
    lib = _load()
    x = _c(x, np.float64)
    flat = x.reshape(-1)
    n = flat.size
    b = n if block is None else int(block)
    out = np.empty(n, np.float64)
    scales = np.empty((n + b - 1) // b, np.float64)
    lib.o_fake_quant(_p(flat), n, b, bits, 1 if symmetric else 0, _p(out), _p(scales))
    return out.reshape(x.shape), scales


def rel_error(ref, approx) -> float:
    """||ref - approx|| / ||ref|| (Frobenius), "Quantize, then dequantize"."""
    ref = np.asarray(ref, np.float64)
    approx = np.asarray(approx, np.float64)
    return float(np.linalg.norm(ref - approx) / np.linalg.norm(ref))


def bits_per_weight(bits: int, symmetric: bool, block: int) -> float:
    """One 16-bit scale per block plus a ``bits``-wide zero point when asymmetric."""
    return bits + (16 + (0 if symmetric else bits)) / block


def bits_per_weight_16bit_zero(bits: int, block: int) -> float:
    """Tahoma accounting, "Achievement 1": 16-bit scale and 16-bit zero term per block."""
    return bits + (16 + 16) / block
