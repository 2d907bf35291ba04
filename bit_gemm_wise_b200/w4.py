"""Thin ctypes binding of ``libw4.so`` (declared in ``include/w4.h``).

Every function here has the name of the C entry point it calls and only marshals
arguments: torch tensors become device pointers, the current torch CUDA stream becomes the
``cudaStream_t``. All computation happens in the library's CUDA kernels. There is no CPU
path: if the library is missing or a call returns an error, these functions raise.
Tensors must be contiguous CUDA tensors that the caller allocated (helpers at the bottom
allocate outputs of the right shape with torch).
"""
from __future__ import annotations

import ctypes
import os

import torch

W4_OK = 0
W4_SYM, W4_ASYM = 0, 1
W4_LAYOUT_GEMV, W4_LAYOUT_GEMM, W4_LAYOUT_TC = 0, 1, 2
W4_OUT_FP32, W4_OVERLAP_PREVIOUS = 1, 2  # flags of w4a16_gemv

STATUS = {
    0: "W4_OK", 1: "W4_ERR_NULL", 2: "W4_ERR_SHAPE", 3: "W4_ERR_GROUP", 4: "W4_ERR_ALIGN",
    5: "W4_ERR_ARG", 6: "W4_ERR_UNSUPPORTED", 7: "W4_ERR_CUDA", 8: "W4_ERR_TIMEOUT",
    9: "W4_ERR_DEVICE_CHECK", 10: "W4_ERR_WORKSPACE", 11: "W4_ERR_SCRATCH_LIMIT",
}

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libw4.so")

# (name, restype, argtypes) of every exported entry point
_P, _I64, _I, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = [
    ("w4_status_str", ctypes.c_char_p, [_I]),
    ("w4_version", _I, []),
    ("w4_quantize", _I, [_P, _I64, _I64, _I, _I, _P, _I, _P, _P, _P, _P, _P]),
    ("w4_prepack_bytes", _SZ, [_I64, _I64, _I, _I]),
    ("w4_prepack", _I, [_P, _P, _P, _I64, _I64, _I, _I, _I, _P, _P]),
    ("w4a8_gsum_op_cols", _I64, [_I64, _I]),
    ("fp8_row_quant", _I, [_P, _I64, _I64, _I, _P, _P, _P, _P, _P, _P]),
    ("fp8_row_quant_gather", _I, [_P, _I64, _I64, _I, _P, _I64, _P, _P, _P, _P, _P, _P]),
    ("w4_moe_route_workspace_bytes", _I64, [_I64, _I]),
    ("w4_moe_route", _I, [_P, _I64, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    ("w4_moe_swiglu_quant", _I, [_P, _I64, _I64, _I, _P, _P, _P, _P, _P]),
    ("w4_moe_combine", _I, [_P, _I64, _I64, _P, _P, _I64, _I, _P, _P]),
    ("w4_nf4_levels", _I, [_P]),
    ("w4_nf4_quantize", _I, [_P, _I64, _I64, _P, _P, _P]),
    ("w4_nf4_gemv", _I, [_P, _I64, _P, _P, _I64, _I64, _P, _I, _P]),
    ("w4a16_gemv_workspace_bytes", _SZ, [_I64, _I64, _I]),
    ("w4a16_gemv_schedule", _I, [_I64, _I64, _I64, _I, _I, _P]),
    ("w4a16_gemv", _I, [_P, _I64, _P, _I64, _I64, _I, _I, _P, _I, _P, _SZ, _P]),
    ("w4a16_gemm_tc_workspace_bytes", _SZ, [_I64, _I64, _I]),
    ("w4a16_gemm_tc_schedule", _I, [_I64, _I64, _I64, _I, _I, _P]),
    ("w4a16_gemm_tc", _I, [_P, _I64, _P, _I64, _I64, _I, _I, _P, _I, _P, _SZ, _P]),
    ("w4a16_gemv_prefetch_next", _I, [_P, _I64, _P, _I64, _I64, _I, _I, _P, _I, _P, _SZ, _P, _SZ, _P]),
    ("w4a16_gemv_noalloc_scratch_limit", _SZ, []),
    ("w4a16_gemv_grouped", _I, [_I, _P, _I64, _P, _P, _P, _I, _I, _P, _I, _P]),
    ("w4a16_gemv_grouped_schedule", _I, [_I, _I64, _P, _P, _I, _I, _P]),
    ("w4a16_gemv_noalloc", _I, [_P, _I64, _P, _I64, _I64, _I, _I, _P, _I, _P]),
    ("w4a8_gemm", _I, [_P, _P, _P, _P, _I64, _P, _I64, _I64, _I, _I, _P, _I, _P, _SZ, _P]),
    ("w4a8_gemm_workspace_bytes", _SZ, [_I64, _I64, _I64, _I]),
    ("w4a8_gemm_schedule", _I, [_I64, _I64, _I64, _I, _I, _P]),
    ("w4a8_gemm_split_segment", _I, [_I64, _I64, _I64, _I64, _I, _P]),
    ("w4a8_gemm_rowquant_workspace_bytes", _SZ, [_I64, _I64, _I64, _I]),
    ("w4a8_gemm_rowquant_layout", _I, [_I64, _I64, _I64, _I, _P]),
    ("w4a8_gemm_rowquant", _I, [_P, _I64, _P, _I64, _I64, _I, _I, _P, _I, _P, _SZ, _P]),
    ("w4a8_grouped_gemm", _I, [_P, _P, _P, _P, _P, _I, _I64, _P, _I64, _I64, _I, _I, _P, _P]),
    ("w4_device_status", _I, [_P, ctypes.POINTER(ctypes.c_int)]),
    ("w4_selftest_bounded_wait", _I, [_I64, _P]),
]

_lib = None


class W4Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn}: {STATUS.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """Load the CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with python -m bit_gemm_wise_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != W4_OK:
        raise W4Error(fn, rc)


def _mode(mode) -> int:
    if mode in ("sym", W4_SYM):
        return W4_SYM
    if mode in ("asym", W4_ASYM):
        return W4_ASYM
    return int(mode)


# ------------------------------------------------------------------ entry points

def w4_status_str(code: int) -> str:
    return lib().w4_status_str(code).decode()


def w4_version() -> int:
    return lib().w4_version()


def w4_quantize(W, N, K, group, mode, clip_grid, codes, scales, zeros=None, chosen=None, stream=None):
    grid = (ctypes.c_float * len(clip_grid))(*[float(r) for r in clip_grid])
    rc = lib().w4_quantize(_ptr(W), N, K, group, _mode(mode), ctypes.cast(grid, _P), len(clip_grid),
                           _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(chosen), _stream(stream))
    _check("w4_quantize", rc)


def w4_prepack_bytes(N, K, group, layout) -> int:
    return int(lib().w4_prepack_bytes(N, K, group, layout))


def w4_prepack(codes, scales, zeros, N, K, group, mode, layout, packed, stream=None):
    rc = lib().w4_prepack(_ptr(codes), _ptr(scales), _ptr(zeros), N, K, group, _mode(mode), layout,
                          _ptr(packed), _stream(stream))
    _check("w4_prepack", rc)


def w4a8_gsum_op_cols(K, group) -> int:
    return int(lib().w4a8_gsum_op_cols(K, group))


def fp8_row_quant(X, M, K, group, X8, row_scale, group_sums=None, gsum_op=None, stream=None, *, x16=None):
    """x16: optional fp16 [M, K] copy of the E4M3 values (the operand of w4a8_gemm at groups
    32 and 256); X8 may then be None."""
    rc = lib().fp8_row_quant(_ptr(X), M, K, group, _ptr(X8), _ptr(row_scale), _ptr(group_sums), _ptr(gsum_op),
                             _ptr(x16), _stream(stream))
    _check("fp8_row_quant", rc)


def fp8_row_quant_gather(X, M_src, K, group, row_index, M, X8, row_scale, group_sums=None, gsum_op=None,
                         stream=None, *, x16=None):
    rc = lib().fp8_row_quant_gather(_ptr(X), M_src, K, group, _ptr(row_index), M, _ptr(X8), _ptr(row_scale),
                                    _ptr(group_sums), _ptr(gsum_op), _ptr(x16), _stream(stream))
    _check("fp8_row_quant_gather", rc)


def w4_moe_route_workspace_bytes(T, E):
    return int(lib().w4_moe_route_workspace_bytes(T, E))


def alloc_moe_route_workspace(T, E, device=None):
    n = w4_moe_route_workspace_bytes(T, E)
    return torch.empty(max(n, 4), dtype=torch.uint8, device=device)


def w4_moe_route(logits, T, E, k, experts, gates, expert_row_offsets, token_of_row, row_of, workspace,
                 stream=None):
    rc = lib().w4_moe_route(_ptr(logits), T, E, k, _ptr(experts), _ptr(gates), _ptr(expert_row_offsets),
                            _ptr(token_of_row), _ptr(row_of), _ptr(workspace), workspace.numel(),
                            _stream(stream))
    _check("w4_moe_route", rc)


def w4_moe_swiglu_quant(gate_up, R, H, group, X8, row_scale, gsum_op=None, stream=None, *, x16=None):
    rc = lib().w4_moe_swiglu_quant(_ptr(gate_up), R, H, group, _ptr(X8), _ptr(row_scale), _ptr(gsum_op), _ptr(x16),
                                   _stream(stream))
    _check("w4_moe_swiglu_quant", rc)


def w4_moe_combine(rows, N, R, row_of, gates, T, k, y, stream=None):
    rc = lib().w4_moe_combine(_ptr(rows), N, R, _ptr(row_of), _ptr(gates), T, k, _ptr(y), _stream(stream))
    _check("w4_moe_combine", rc)


def w4_nf4_levels():
    out = (ctypes.c_float * 16)()
    _check("w4_nf4_levels", lib().w4_nf4_levels(ctypes.cast(out, _P)))
    return [float(v) for v in out]


def w4_nf4_quantize(W, N, K, codes, absmax, stream=None):
    _check("w4_nf4_quantize", lib().w4_nf4_quantize(_ptr(W), N, K, _ptr(codes), _ptr(absmax), _stream(stream)))


def w4_nf4_gemv(x, M, codes, absmax, N, K, y, flags=0, stream=None):
    rc = lib().w4_nf4_gemv(_ptr(x), M, _ptr(codes), _ptr(absmax), N, K, _ptr(y), int(flags), _stream(stream))
    _check("w4_nf4_gemv", rc)


def w4a16_gemv_workspace_bytes(N, K, group) -> int:
    return int(lib().w4a16_gemv_workspace_bytes(N, K, group))


def w4a16_gemv_schedule(M, N, K, group, sms) -> dict:
    """Host-only: how w4a16_gemv divides the problem over `sms` SMs."""
    out = (ctypes.c_int64 * 8)()
    _check("w4a16_gemv_schedule", lib().w4a16_gemv_schedule(M, N, K, group, sms, out))
    keys = ("rows_per_sweep", "sweeps", "k_parts", "row_blocks", "rows_per_block", "smem_bytes", "stages",
            "workspace_bytes")
    return dict(zip(keys, (int(v) for v in out)))


def w4a16_gemv(x, M, packed, N, K, group, mode, y, flags, workspace, stream=None):
    """flags: W4_OUT_FP32 (fp32 y) | W4_OVERLAP_PREVIOUS (programmatic dependent launch)."""
    rc = lib().w4a16_gemv(_ptr(x), M, _ptr(packed), N, K, group, _mode(mode), _ptr(y), int(flags),
                          _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                          _stream(stream))
    _check("w4a16_gemv", rc)


def w4a16_gemm_tc_workspace_bytes(N, K, group) -> int:
    return int(lib().w4a16_gemm_tc_workspace_bytes(N, K, group))


def w4a16_gemm_tc_schedule(M, N, K, group, sms) -> dict:
    """Host-only: how w4a16_gemm_tc divides the problem over `sms` SMs."""
    out = (ctypes.c_int64 * 6)()
    _check("w4a16_gemm_tc_schedule", lib().w4a16_gemm_tc_schedule(M, N, K, group, sms, out))
    keys = ("tiles", "k_blocks", "units", "ctas", "k_per_block", "record_bytes")
    return dict(zip(keys, (int(v) for v in out)))


def w4a16_gemm_tc(x, M, packed, N, K, group, mode, y, flags, workspace, stream=None):
    """Tensor-core W4A16 for 1 <= M <= 16 (packed: W4_LAYOUT_TC); flags as w4a16_gemv."""
    rc = lib().w4a16_gemm_tc(_ptr(x), M, _ptr(packed), N, K, group, _mode(mode), _ptr(y), int(flags),
                             _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                             _stream(stream))
    _check("w4a16_gemm_tc", rc)


def w4a16_gemv_prefetch_next(x, M, packed, N, K, group, mode, y, flags, workspace, next_packed, next_bytes=None,
                             stream=None):
    """w4a16_gemv that also brings next_bytes bytes at next_packed (the weights of the GEMV that
    follows on the stream) into L2 once each block's own rows are requested."""
    if next_bytes is None:
        next_bytes = 0 if next_packed is None else next_packed.numel() * next_packed.element_size()
    rc = lib().w4a16_gemv_prefetch_next(_ptr(x), M, _ptr(packed), N, K, group, _mode(mode), _ptr(y), int(flags),
                                        _ptr(workspace),
                                        0 if workspace is None else workspace.numel() * workspace.element_size(),
                                        _ptr(next_packed), int(next_bytes), _stream(stream))
    _check("w4a16_gemv_prefetch_next", rc)


def w4a16_gemv_grouped(xs, M, packeds, Ns, Ks, group, mode, ys, flags, stream=None):
    """Independent GEMVs (same M, group, mode) in one launch; lists of tensors and sizes."""
    n = len(xs)
    P = ctypes.c_void_p * n
    L = ctypes.c_int64 * n
    rc = lib().w4a16_gemv_grouped(n, P(*[_ptr(t) for t in xs]), M, P(*[_ptr(t) for t in packeds]),
                                  L(*Ns), L(*Ks), group, _mode(mode), P(*[_ptr(t) for t in ys]), int(flags),
                                  _stream(stream))
    _check("w4a16_gemv_grouped", rc)


def w4a16_gemv_grouped_schedule(M, Ns, Ks, group, sms):
    """Host-only: blocks per problem of a grouped launch on `sms` SMs."""
    n = len(Ns)
    out = (ctypes.c_int64 * n)()
    L = ctypes.c_int64 * n
    _check("w4a16_gemv_grouped_schedule",
           lib().w4a16_gemv_grouped_schedule(n, M, L(*Ns), L(*Ks), group, sms, ctypes.cast(out, _P)))
    return [int(v) for v in out]


def w4a16_gemv_noalloc_scratch_limit() -> int:
    return int(lib().w4a16_gemv_noalloc_scratch_limit())


def w4a16_gemv_noalloc(x, M, packed, N, K, group, mode, y, flags, stream=None):
    """w4a16_gemv with the library's fixed scratch array instead of a caller workspace."""
    rc = lib().w4a16_gemv_noalloc(_ptr(x), M, _ptr(packed), N, K, group, _mode(mode), _ptr(y), int(flags),
                                  _stream(stream))
    _check("w4a16_gemv_noalloc", rc)


def w4a8_gemm(X8, row_scale, gsum_op, M, packed, N, K, group, mode, Y, out_fp32=0, workspace=None, stream=None,
              *, X16=None):
    """workspace: None (every tile whole) or alloc_gemm_workspace(M, N, K, group) (the last
    wave's tiles may be split along K). Groups 64 and 128 take X8 and gsum_op, groups 32 and
    256 take X16 (fp8_row_quant's fp16 copy of the E4M3 values)."""
    rc = lib().w4a8_gemm(_ptr(X8), _ptr(X16), _ptr(row_scale), _ptr(gsum_op), M, _ptr(packed), N, K, group,
                         _mode(mode), _ptr(Y), int(out_fp32), _ptr(workspace),
                         0 if workspace is None else workspace.numel() * workspace.element_size(),
                         _stream(stream))
    _check("w4a8_gemm", rc)


def w4a8_gemm_rowquant(X, M, packed, N, K, group, mode, Y, out_fp32, workspace, stream=None):
    """Row quant and W4A8 GEMM in one launch from bf16 activations X [M, K]; workspace:
    alloc_gemm_rowquant_workspace(M, N, K, group) (groups 64 and 128)."""
    rc = lib().w4a8_gemm_rowquant(_ptr(X), M, _ptr(packed), N, K, group, _mode(mode), _ptr(Y), int(out_fp32),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check("w4a8_gemm_rowquant", rc)


def w4a8_gemm_rowquant_workspace_bytes(M, N, K, group) -> int:
    return int(lib().w4a8_gemm_rowquant_workspace_bytes(M, N, K, group))


def w4a8_gemm_rowquant_layout(M, N, K, group) -> dict:
    """Host-only: byte offsets of the E4M3 rows, row scales and group-sum operand that
    w4a8_gemm_rowquant leaves in its workspace, and the workspace size."""
    out = (ctypes.c_int64 * 4)()
    _check("w4a8_gemm_rowquant_layout", lib().w4a8_gemm_rowquant_layout(M, N, K, group, out))
    return dict(zip(("X_e4m3", "row_scale", "gsum_op", "bytes"), (int(v) for v in out)))


def w4a8_gemm_workspace_bytes(M, N, K, group) -> int:
    return int(lib().w4a8_gemm_workspace_bytes(M, N, K, group))


def w4a8_gemm_schedule(M, N, K, group, sms) -> dict:
    """Host-only: how w4a8_gemm with a workspace divides the problem over `sms` SMs."""
    out = (ctypes.c_int64 * 7)()
    _check("w4a8_gemm_schedule", lib().w4a8_gemm_schedule(M, N, K, group, sms, out))
    keys = ("tiles", "whole_tiles", "split_tiles", "split_blocks", "grid", "workspace_bytes", "k_blocks")
    return dict(zip(keys, (int(v) for v in out)))


def w4a8_gemm_split_segment(R, KT, PS, c, s):
    """Host-only: segment s of block c among PS blocks sharing R split tiles of KT k-blocks:
    None, or (tile, kb0, kb1, first_block, last_block, slot)."""
    out = (ctypes.c_int64 * 7)()
    _check("w4a8_gemm_split_segment", lib().w4a8_gemm_split_segment(R, KT, PS, c, s, out))
    return None if out[0] == 0 else tuple(int(v) for v in out[1:])


def w4a8_grouped_gemm(X8, row_scale, gsum_op, expert_row_offsets, E, M_total, packed, N, K, group,
                      mode, Y, stream=None, *, X16=None):
    rc = lib().w4a8_grouped_gemm(_ptr(X8), _ptr(X16), _ptr(row_scale), _ptr(gsum_op), _ptr(expert_row_offsets), E,
                                 M_total, _ptr(packed), N, K, group, _mode(mode), _ptr(Y), _stream(stream))
    _check("w4a8_grouped_gemm", rc)


def w4_device_status(stream=None) -> int:
    code = ctypes.c_int(-1)
    rc = lib().w4_device_status(_stream(stream), ctypes.byref(code))
    _check("w4_device_status", rc)
    return code.value


def w4_selftest_bounded_wait(limit_ns, stream=None):
    """Launch a bounded wait that must expire (diagnostic of the kernels' failure path)."""
    _check("w4_selftest_bounded_wait", lib().w4_selftest_bounded_wait(int(limit_ns), _stream(stream)))


# ------------------------------------------------------------------ allocation helpers

def alloc_quantized(N, K, group, mode, device="cuda", chosen=True):
    """Empty canonical outputs of w4_quantize: codes u8 [N,K/2], scales fp16 bits [N,K/g],
    zeros int16 [N,K/g] (asym only), chosen u8 [N,K/g] (optional)."""
    J = K // group
    codes = torch.empty(N, K // 2, dtype=torch.uint8, device=device)
    scales = torch.empty(N, J, dtype=torch.int16, device=device)
    zeros = torch.empty(N, J, dtype=torch.int16, device=device) if _mode(mode) == W4_ASYM else None
    ch = torch.empty(N, J, dtype=torch.uint8, device=device) if chosen else None
    return codes, scales, zeros, ch


def alloc_gemv_workspace(N, K, group, device="cuda"):
    """Zero-filled workspace for w4a16_gemv (calls leave it zero-filled), or None when no
    call of this shape needs one (rows short enough for one block)."""
    nbytes = w4a16_gemv_workspace_bytes(N, K, group)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device) if nbytes else None


def alloc_tc_workspace(N, K, group, device="cuda"):
    """Zero-filled workspace for w4a16_gemm_tc (calls leave its counters zero)."""
    nbytes = w4a16_gemm_tc_workspace_bytes(N, K, group)
    if nbytes == 0:
        raise W4Error("w4a16_gemm_tc_workspace_bytes", 2)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def alloc_gemm_workspace(M, N, K, group, device="cuda"):
    """Zero-filled workspace for w4a8_gemm, or None when the shape is never split."""
    nbytes = w4a8_gemm_workspace_bytes(M, N, K, group)
    return torch.zeros(nbytes, dtype=torch.uint8, device=device) if nbytes else None


def alloc_gemm_rowquant_workspace(M, N, K, group, device="cuda"):
    """Workspace for w4a8_gemm_rowquant (uninitialised: every call clears what it needs)."""
    nbytes = w4a8_gemm_rowquant_workspace_bytes(M, N, K, group)
    if nbytes == 0:
        raise W4Error("w4a8_gemm_rowquant_workspace_bytes", 6)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def alloc_packed(N, K, group, layout, device="cuda", copies: int = 1):
    nbytes = w4_prepack_bytes(N, K, group, layout)
    if nbytes == 0:
        raise W4Error("w4_prepack_bytes", 2)
    return torch.empty(copies * nbytes, dtype=torch.uint8, device=device)


def alloc_row_quant(M, K, group, device="cuda", group_sums=True):
    """Empty outputs of fp8_row_quant for the W4A8 GEMM: X8 u8 [M,K], row scales fp32 [M],
    group sums fp32 [M,K/g] (optional) and the GEMM's group-sum operand bf16 [M, cols]."""
    cols = w4a8_gsum_op_cols(K, group)
    if cols == 0:
        raise W4Error("w4a8_gsum_op_cols", 3)
    X8 = torch.empty(M, K, dtype=torch.uint8, device=device)
    sa = torch.empty(M, dtype=torch.float32, device=device)
    G = torch.empty(M, K // group, dtype=torch.float32, device=device) if group_sums else None
    gop = torch.empty(M, cols, dtype=torch.bfloat16, device=device)
    return X8, sa, G, gop
