"""Column-parallel OPQ linear over torch.distributed ranks (one process per GPU).

The rows of W[N, K] (output features) are independent under OPQ: each row carries its own
max, codes and signs ("OPQ INT4 Z-Image" model card, "OPQ principle" and "storage format").
So a weight splits into contiguous row shards, one per rank; each rank quantizes its own
shard and computes its slice y[:, lo:hi] = x W'[lo:hi]^T with the packed-weight linear, and
one all-gather along N assembles y on every rank (x replicated). Shards differ in size by at
most one row; the gather moves equal-width blocks (the shorter ones padded) and the padding
is dropped on reassembly.

Only the plumbing lives here: the quantize and the local linear are the library's kernels
(``opq.quantize`` / ``opq.linear``), the exchange is ``torch.distributed`` (NCCL between
GPUs). ``linear_fn`` can be replaced (same signature as ``opq.linear`` without the keyword
arguments) to drive the exchange logic with another implementation of the local product.
"""
from dataclasses import dataclass
from typing import Callable, Optional

import torch
import torch.distributed as dist


def shard_range(n_rows: int, rank: int, world: int):
    """Contiguous row range [lo, hi) of ``rank``: the first n_rows % world ranks take one more row."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world {world}")
    base, rem = divmod(n_rows, world)
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def shard_layers(n_layers: int, rank: int, world: int):
    """Layers of ``rank`` in a whole-model quantize pass: round-robin, so that every rank gets
    the same mix of matrix shapes (layers are independent under OPQ)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} out of range for world {world}")
    return list(range(rank, n_layers, world))


def shard_width(n_rows: int, world: int) -> int:
    """Width of the gathered blocks: the largest shard."""
    return -(-n_rows // world)


@dataclass
class ColumnShard:
    """One rank's packed rows [lo, hi) of a per-row OPQ weight with N rows."""
    codes: torch.Tensor      # int32 [hi - lo, K / 8]
    signs: torch.Tensor      # int32 [hi - lo, K / 32]
    scales: torch.Tensor     # float32 [hi - lo]
    lo: int
    hi: int
    n_rows: int
    alpha: float


def quantize_shard(w: torch.Tensor, rank: int, world: int, alpha: Optional[float] = None,
                   quantize_fn: Optional[Callable] = None) -> ColumnShard:
    """Quantize this rank's rows of bf16 W[N, K] (W may be the full matrix or any view of it)."""
    from . import ALPHA, quantize
    alpha = ALPHA if alpha is None else alpha
    quantize_fn = quantize if quantize_fn is None else quantize_fn
    lo, hi = shard_range(w.shape[0], rank, world)
    if hi == lo:
        raise ValueError("empty shard: fewer rows than ranks")
    codes, signs, scales = quantize_fn(w[lo:hi].contiguous(), alpha)
    return ColumnShard(codes, signs, scales, lo, hi, w.shape[0], alpha)


def column_parallel_linear(x: torch.Tensor, shard: ColumnShard, group=None, out: Optional[torch.Tensor] = None,
                           linear_fn: Optional[Callable] = None) -> torch.Tensor:
    """y[M, N] = x W'^T on every rank of ``group`` from the local shard and one all-gather.

    Every rank passes the same x[M, K] and its own shard; all ranks take the same collective
    steps in the same order."""
    from . import linear
    linear_fn = linear if linear_fn is None else linear_fn
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    lo, hi = shard_range(shard.n_rows, rank, world)
    if (lo, hi) != (shard.lo, shard.hi):
        raise ValueError(f"shard rows [{shard.lo}, {shard.hi}) do not belong to rank {rank} of {world}")
    M = x.shape[0]
    S = shard_width(shard.n_rows, world)
    y_local = linear_fn(x, shard.codes, shard.signs, shard.scales, shard.alpha)     # [M, hi - lo]
    # equal-width blocks, rank-major: block r holds y[:, lo_r:hi_r] in its first hi_r - lo_r columns
    send = torch.zeros((M, S), dtype=y_local.dtype, device=y_local.device)
    send[:, :hi - lo] = y_local
    gathered = torch.empty((world * M, S), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(gathered, send, group=group)
    blocks = gathered.view(world, M, S)
    y = out if out is not None else torch.empty((M, shard.n_rows), dtype=y_local.dtype, device=y_local.device)
    for r in range(world):
        a, b = shard_range(shard.n_rows, r, world)
        y[:, a:b] = blocks[r, :, :b - a]
    return y
