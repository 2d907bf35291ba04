"""Column-parallel split of a quantized linear layer over the ranks of one node.

The weight W[N, K] is cut along N (the output features): every rank owns a contiguous run of
rows, quantizes, prepacks and multiplies them on its own GPU, and produces y[:, n0:n1] with
no exchange inside any kernel. Each row's groups and each output's dot product involve only
that row, so the concatenation of the ranks' slices equals the unsplit result exactly. Where
the next operation needs all of y, an all_gather over NCCL joins the slices in rank order.
"""
from __future__ import annotations

GEMM_TILE_ROWS = 128  # weight rows per tile of the W4A8 GEMM


def column_shard(N: int, world: int, rank: int, granule: int = GEMM_TILE_ROWS) -> tuple[int, int]:
    """Rows [n0, n1) of W[N, K] owned by `rank` of `world`: whole granules (the GEMM's
    128-row weight tiles by default; 1 for the GEMV, which takes any row range), spread as
    evenly as the granules allow, ranks in order. A rank may own no row when N has fewer
    granules than there are ranks."""
    if world < 1 or not 0 <= rank < world or N < 0 or granule < 1:
        raise ValueError(f"column_shard: N={N} world={world} rank={rank} granule={granule}")
    units = (N + granule - 1) // granule
    lo = rank * units // world
    hi = (rank + 1) * units // world
    return min(N, lo * granule), min(N, hi * granule)
