"""Row split of a quantized linear across ranks (one process per GPU).

Every row of W is quantized on its own: groups run along K inside one row
(metalworking "MLX Quantization", section "Mechanics"; "Quantizing a Model for
MLX", section "What MLX quantization stores").  So W[N, K] splits along N into
contiguous row ranges with no change to the packed format: rank r holds rows
[n0, n1) of ``packed``, ``scales`` and ``biases`` (a contiguous slice of each),
computes y[:, n0:n1] = x @ dequant(W[n0:n1])^T with no exchange, and, when a
replicated y is wanted, one all-gather of y (M * N * 2 bytes) assembles it.

This module is host plumbing only: the slicing of caller tensors and the
collective.  The product itself is ``aq_matmul`` on the rank's slice.
"""
from __future__ import annotations

import torch

# Row ranges start on multiples of 16 rows: the tensor-core decode kernel takes
# W in 16-row tiles, and a 16-row boundary keeps every slice's packed rows,
# scales and biases 16-byte aligned whenever the whole arrays are.
ROW_ALIGN = 16


def row_range(N: int, world: int, rank: int, align: int = ROW_ALIGN) -> tuple[int, int]:
    """Rows [n0, n1) of rank ``rank`` out of ``world``: contiguous, in rank order,
    covering [0, N) exactly once, sizes differing by at most ``align`` rows (the
    last ranks may get none when N is small)."""
    if world < 1 or not 0 <= rank < world or N < 0:
        raise ValueError(f"bad split: N={N} world={world} rank={rank}")
    units = -(-N // align)  # align-row units, the last one possibly short
    u0 = units * rank // world
    u1 = units * (rank + 1) // world
    return min(N, u0 * align), min(N, u1 * align)


def shard_rows(packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, world: int, rank: int):
    """This rank's rows of a quantized W (views, no copy): (packed, scales, biases, n0, n1)."""
    N = packed.shape[0]
    if scales.shape[0] != N or biases.shape[0] != N:
        raise ValueError("packed, scales and biases must have the same number of rows")
    n0, n1 = row_range(N, world, rank)
    return packed[n0:n1], scales[n0:n1], biases[n0:n1], n0, n1


def all_gather_columns(y_local: torch.Tensor, N: int, group=None) -> torch.Tensor:
    """Assemble y[M, N] from every rank's y[:, n0:n1] (row_range's split) with one
    all-gather.  Slices are padded to the largest one so that the collective moves
    equal blocks; the padding is dropped on assembly."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    M = y_local.shape[0]
    ranges = [row_range(N, world, r) for r in range(world)]
    width = max(n1 - n0 for n0, n1 in ranges)
    n0, n1 = ranges[rank]
    if y_local.shape != (M, n1 - n0):
        raise ValueError(f"rank {rank} holds y of shape {tuple(y_local.shape)}, expected {(M, n1 - n0)}")
    send = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
    send[:, : n1 - n0] = y_local
    recv = [torch.empty((M, width), dtype=y_local.dtype, device=y_local.device) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    return torch.cat([recv[r][:, : b - a] for r, (a, b) in enumerate(ranges)], dim=1)


def sharded_matmul(x: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, biases: torch.Tensor, G: int,
                   bits: int, N: int, group=None, gather: bool = True, **kw) -> torch.Tensor:
    """y = x @ dequant(W)^T with W split along N over the ranks of ``group``.

    ``packed``/``scales``/``biases`` are this rank's rows (``shard_rows``) of a W
    with ``N`` rows in total.  Each rank runs ``aq_matmul`` on its rows; with
    ``gather`` the full y[M, N] is assembled by one all-gather, else the local
    y[:, n0:n1] is returned."""
    import torch.distributed as dist

    from . import aq_matmul
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    n0, n1 = row_range(N, world, rank)
    if packed.shape[0] != n1 - n0:
        raise ValueError(f"rank {rank} holds {packed.shape[0]} rows, its range is [{n0}, {n1})")
    if n1 > n0:
        y_local = aq_matmul(x, packed, scales, biases, G, bits, **kw)
    else:
        y_local = torch.empty((x.shape[0], 0), dtype=torch.bfloat16, device=x.device)
    return all_gather_columns(y_local, N, group) if gather else y_local
