"""Seeded synthetic inputs for every workload of the path.

This module is the only code shared by the CUDA path and the CPU oracle. It draws random
numbers and lays out shapes; it contains none of the quantizer, activation-quantizer or
matmul arithmetic. Every tensor comes from its own ``torch.Generator`` seeded with
``seed * 1000 + tensor_index``. Normals are drawn in fp32 and rounded to bf16 (RN).

Workloads (shapes follow the pages' layers; values are synthetic stand-ins for the real
checkpoints, activations and datasets the pages measure on):

* ``single_layer``  -- "Quantizing LLMs in practice", One real weight matrix: a 576x1536
  down_proj layer. W[N=1536, K=576] ~ N(0, 0.02) with 4 whole input columns x50, x[1,576] ~ N(0,1).
  Symmetric INT4, group 32, clip grid {1.0}.
* ``decode_sweep``  -- 8B-model decode GEMV shapes (K,N) in {(4096,4096),(4096,1024),
  (4096,14336),(14336,4096)}; W ~ N(0, 0.02) with round(0.001*K) outlier input columns x30;
  asymmetric group 128 with the 20-ratio clip grid; x[M,K] ~ N(0,1), M in {1,4,16}.
* ``prefill_gemm``  -- W4A8 prefill: M=4096 tokens, (K,N) in {(3840,15360),(15360,3840)};
  W ~ N(0, 0.02); X ~ N(0,1) with 8 outlier columns x20; asymmetric group 128, grid {1.0}.
* ``weight_set_8b`` -- Llama-3.1-8B block weights ("Quantizing LLMs in practice", memory
  calculator): per layer q,o [4096,4096], k,v [1024,4096], gate,up [14336,4096],
  down [4096,14336]; 32 layers. W = 0.02 * T / sqrt(3), T ~ Student-t(3).
* ``moe_experts``   -- 32 experts, gate_up [5760,2880] and down [2880,2880], group 32 asym;
  4096 tokens X ~ N(0,1) routed top-4 by U(0,1) logits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

BF16 = torch.bfloat16


def _gen(seed: int, index: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + index)
    return g


def normal(shape, std: float, seed: int, index: int, device="cpu") -> torch.Tensor:
    """fp32 N(0, std) rounded to bf16."""
    g = _gen(seed, index, device)
    return (torch.randn(*shape, generator=g, device=device) * std).to(BF16)


def clip_grid_20() -> list[float]:
    """20 clip ratios evenly spaced over [0.7, 1.0], largest first: r_i = 1 - 0.3*i/19,
    formed in double precision and rounded to fp32 once. grid[0] == 1.0 exactly."""
    return [float(torch.tensor(1.0 - 0.3 * i / 19.0, dtype=torch.float32)) for i in range(20)]


def clip_grid_page() -> list[float]:
    """The 11 contracted ranges of the Tahoma post, "MSE clipping" (1.00, 0.95, ..., 0.50)."""
    return [float(torch.tensor(1.0 - 0.05 * i, dtype=torch.float32)) for i in range(11)]


def outlier_weight(N: int, K: int, n_cols: int, factor: float, seed: int, index: int,
                   std: float = 0.02, device="cpu") -> torch.Tensor:
    """W[N,K] ~ N(0,std) with ``n_cols`` whole input columns (drawn by randperm) scaled by
    ``factor`` before the bf16 rounding."""
    g = _gen(seed, index, device)
    w = torch.randn(N, K, generator=g, device=device) * std
    if n_cols:
        gc = _gen(seed, index + 500, "cpu")
        cols = torch.randperm(K, generator=gc)[:n_cols].to(device)
        w[:, cols] *= factor
    return w.to(BF16)


def outlier_activation(M: int, K: int, n_cols: int, factor: float, seed: int, index: int,
                       device="cpu") -> torch.Tensor:
    g = _gen(seed, index, device)
    x = torch.randn(M, K, generator=g, device=device)
    if n_cols:
        gc = _gen(seed, index + 500, "cpu")
        cols = torch.randperm(K, generator=gc)[:n_cols].to(device)
        x[:, cols] *= factor
    return x.to(BF16)


def student_t3_weight(N: int, K: int, seed: int, index: int, device="cpu",
                      std: float = 0.02) -> torch.Tensor:
    """W = std * T / sqrt(3) with T ~ Student-t(nu=3) = Z / sqrt(V/3), V ~ chi^2(3)."""
    g = _gen(seed, index, device)
    z = torch.randn(N, K, generator=g, device=device)
    v = torch.zeros(N, K, device=device)
    for _ in range(3):
        v += torch.randn(N, K, generator=g, device=device).square_()
    t = z / torch.sqrt(v / 3.0)
    return (t * (std / math.sqrt(3.0))).to(BF16)


# ---------------------------------------------------------------- workloads

SINGLE_LAYER = dict(N=1536, K=576, group=32, mode="sym", outlier_cols=4, outlier_factor=50.0)

DECODE_SHAPES = [(4096, 4096), (4096, 1024), (4096, 14336), (14336, 4096)]  # (K, N)
DECODE_M = (1, 4, 16)

PREFILL_M = 4096
PREFILL_SHAPES = [(3840, 15360), (15360, 3840)]  # (K, N)

LLAMA8B_LAYER = [  # (name, N, K)
    ("q", 4096, 4096), ("k", 1024, 4096), ("v", 1024, 4096), ("o", 4096, 4096),
    ("gate", 14336, 4096), ("up", 14336, 4096), ("down", 4096, 14336),
]
LLAMA8B_LAYERS = 32

MOE = dict(E=32, top_k=4, tokens=4096, K=2880, N_gate_up=5760, N_down=2880, group=32)


def single_layer(seed: int = 0, device="cpu"):
    c = SINGLE_LAYER
    W = outlier_weight(c["N"], c["K"], c["outlier_cols"], c["outlier_factor"], seed, 0, device=device)
    x = normal((1, c["K"]), 1.0, seed, 1, device=device)
    return W, x


def single_layer_page_orientation(seed: int = 0, device="cpu"):
    """The page's own orientation of the same layer: W[576 out, 1536 in]."""
    W = outlier_weight(576, 1536, 4, 50.0, seed, 2, device=device)
    x = normal((1, 1536), 1.0, seed, 3, device=device)
    return W, x


def decode_weight(K: int, N: int, seed: int = 0, device="cpu"):
    idx = 10 + DECODE_SHAPES.index((K, N)) if (K, N) in DECODE_SHAPES else 19
    return outlier_weight(N, K, int(round(0.001 * K)), 30.0, seed, idx, device=device)


def decode_activation(M: int, K: int, seed: int = 0, device="cpu"):
    return normal((M, K), 1.0, seed, 20 + M, device=device)


def prefill_weight(K: int, N: int, seed: int = 0, device="cpu"):
    return outlier_weight(N, K, 0, 1.0, seed, 40 + (0 if K == 3840 else 1), device=device)


def prefill_activation(M: int, K: int, seed: int = 0, device="cpu"):
    return outlier_activation(M, K, 8, 20.0, seed, 45 + (0 if K == 3840 else 1), device=device)


def llama8b_weight(layer: int, name: str, seed: int = 0, device="cpu"):
    names = [n for n, _, _ in LLAMA8B_LAYER]
    _, N, K = LLAMA8B_LAYER[names.index(name)]
    return student_t3_weight(N, K, seed, 100 + 10 * layer + names.index(name), device=device)


def llama8b_weight_count() -> int:
    return LLAMA8B_LAYERS * sum(N * K for _, N, K in LLAMA8B_LAYER)


@dataclass
class MoeRouting:
    token_of_row: torch.Tensor       # int64 [tokens*top_k]: source token of each grouped row
    expert_row_offsets: torch.Tensor  # int32 [E+1]: rows of expert e are [off[e], off[e+1])


def moe_routing(seed: int = 0) -> MoeRouting:
    """Top-k of U(0,1) logits per token; equal logits go to the lower expert index; rows are
    grouped by expert, tokens ascending inside an expert."""
    c = MOE
    g = _gen(seed, 60)
    logits = torch.rand(c["tokens"], c["E"], generator=g)
    order = torch.sort(-logits, dim=1, stable=True).indices[:, : c["top_k"]]
    chosen = torch.zeros(c["tokens"], c["E"], dtype=torch.bool)
    chosen.scatter_(1, order, True)
    rows, counts = [], []
    for e in range(c["E"]):
        toks = torch.nonzero(chosen[:, e], as_tuple=False).flatten()
        rows.append(toks)
        counts.append(toks.numel())
    off = torch.zeros(c["E"] + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(torch.tensor(counts, dtype=torch.int64), 0).to(torch.int32)
    return MoeRouting(torch.cat(rows), off)


def moe_activation(seed: int = 0, device="cpu"):
    return normal((MOE["tokens"], MOE["K"]), 1.0, seed, 61, device=device)


def moe_weight(kind: str, expert: int, seed: int = 0, device="cpu"):
    N = MOE["N_gate_up"] if kind == "gate_up" else MOE["N_down"]
    return normal((N, MOE["K"]), 0.02, seed, 200 + 2 * expert + (0 if kind == "gate_up" else 1),
                  device=device)


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 array of its bit patterns (CPU)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
