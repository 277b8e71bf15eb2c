"""Tensor-parallel decoder-layer products over several GPUs (one process per GPU).

A layer's products are split the Megatron way: a column-parallel product (fused QKV,
gate+up) gives each rank a contiguous range of output rows, so its input is the full
x and its output stays local; a row-parallel product (O, down) gives each rank a range
of input features, its partial output is summed over the ranks with one all-reduce
(NCCL over NVLink on GPUs). The row ranges are whole groups of four (the packed
storage order), the input-feature ranges whole scale blocks (128 weights; 512, the
rotation block, for the 2-bit format), so a shard packs to exactly the bytes of the
corresponding rows or blocks of the whole matrix. Row-parallel partials are computed
in fp32 (lbq_gemv_f32) and rounded to bf16 once, after the sum, so the result meets
the same 2^-8 * sum|w x| bound as one GPU's product.

This module only plans shards and moves data; every product runs in the library's
kernels. `gemv` and `gemv_f32` may be replaced by callers (the CPU tests of the
planning and the all-reduce pass stand-ins that need no GPU).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

TERN5, SIGN1, Q2RHT = 1, 2, 3


def block_of(fmt: int) -> int:
    """Smallest input-feature split granule: one scale block (the 2-bit format: one
    rotation block, since each rank rotates its own slice of x)."""
    return 512 if fmt == Q2RHT else 128


def split_range(total: int, world: int, rank: int, granule: int) -> tuple[int, int]:
    """Rank `rank`'s [start, end) of `total` items in whole granules, as even as the
    granule allows (the last ranks may get one granule fewer)."""
    assert total % granule == 0 or granule == 4, "input features come in whole blocks"
    units = (total + granule - 1) // granule
    lo = rank * units // world
    hi = (rank + 1) * units // world
    return min(lo * granule, total), min(hi * granule, total)


@dataclass
class Shard:
    kind: str     # "column" or "row"
    fmt: int
    K: int        # the whole matrix's input features
    N: int        # the whole matrix's output features
    lo: int       # this rank's first output row (column) or input feature (row)
    hi: int
    weights: object  # the packed shard (lbq.PackedWeights, or a stand-in)


def make_shard(W: torch.Tensor, fmt: int, kind: str, rank: int, world: int, pack) -> Shard:
    """Cuts rank `rank`'s part out of the fp32 weights W [N][K] and packs it with
    `pack(fmt, W_part)` (lbq.lbq_pack on a GPU)."""
    N, K = W.shape
    if kind == "column":
        lo, hi = split_range(N, world, rank, 4)
        part = W[lo:hi].contiguous()
    elif kind == "row":
        lo, hi = split_range(K, world, rank, block_of(fmt))
        part = W[:, lo:hi].contiguous()
    else:
        raise ValueError(f"unknown split {kind!r}")
    return Shard(kind, fmt, K, N, lo, hi, pack(fmt, part) if hi > lo else None)


def column_forward(shard: Shard, x: torch.Tensor, D=None, gemv=None) -> torch.Tensor:
    """A column-parallel product: this rank's output rows [lo, hi) of W x (bf16)."""
    if gemv is None:
        from . import lbq
        gemv = lbq.lbq_gemv
    return gemv(shard.weights, x, D)


def row_forward(shard: Shard, x: torch.Tensor, D=None, gemv_f32=None, group=None) -> torch.Tensor:
    """A row-parallel product: this rank's partial W[:, lo:hi] x[lo:hi] in fp32, summed
    over the ranks by one all-reduce, then rounded to bf16 once. x is the full input
    (each rank reads its slice); D the full rotation signs (2-bit format)."""
    import torch.distributed as dist
    if gemv_f32 is None:
        from . import lbq
        gemv_f32 = lbq.lbq_gemv_f32
    if shard.weights is not None:
        Ds = None if D is None else D[shard.lo:shard.hi]
        part = gemv_f32(shard.weights, x[shard.lo:shard.hi], Ds).to(torch.float32)
    else:  # more ranks than input blocks: this rank adds nothing
        part = torch.zeros(shard.N, dtype=torch.float32, device=x.device)
    dist.all_reduce(part, op=dist.ReduceOp.SUM, group=group)
    return part.to(torch.bfloat16)


def layer_plan(fmt: int):
    """The split of each product of a decoder layer (fused QKV, O, gate+up, down)."""
    return (("qkv", "column"), ("o", "row"), ("gate_up", "column"), ("down", "row"))
