"""Tensor-parallel MGLU FFN block over the ranks of a torch.distributed group.

The hidden units are split into contiguous shards, one per rank: rank r owns
hidden units [j0, j1), i.e. rows j0..j1-1 of W and of its packed mask bits and
columns j0..j1-1 of W_down.  The up-projection needs no exchange, since output
column j depends only on row j of W and that row's mask bits ("Masked Gated
Linear Unit", "Approach": one weight matrix and its masks, combined per output
unit).  The down-projection then sums over hidden units, so each rank's FFN
block on its shard gives a partial y_r = MGLU_r(x) W_down[:, j0:j1]^T, and one
all-reduce (sum) over the group gives y = sum_r y_r.

Every product runs in the library's kernels (``mglu.forward_down`` on the
shard); this module only slices the weights and calls the collective.  The
partials are bf16 (the library's output type), so y equals the one-GPU block
up to the rounding of each partial and of the reduction: per element at most
about (world + 1) * 2^-8 * sum_r |y_r| apart.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist

from . import mglu

ROW_BLOCK = 16  # shard boundaries fall on the decode kernel's row blocks


def shard_range(h: int, world: int, rank: int, align: int = ROW_BLOCK) -> tuple[int, int]:
    """Hidden units [j0, j1) of `rank`: whole blocks of `align` units split as
    evenly as possible, the first ranks taking one block more; the last rank
    also takes the ragged tail.  Ranks past the number of blocks get none."""
    if world <= 0 or not 0 <= rank < world or h < 0:
        raise ValueError("need 0 <= rank < world and h >= 0")
    blocks = (h + align - 1) // align
    q, r = divmod(blocks, world)
    b0 = rank * q + min(rank, r)
    b1 = b0 + q + (1 if rank < r else 0)
    return min(b0 * align, h), min(b1 * align, h)


@dataclass
class Shard:
    j0: int
    j1: int
    W: torch.Tensor        # [j1 - j0][d], a view of W
    packed: torch.Tensor   # the shard's rows of the packed mask stream, a view
    W_down: torch.Tensor   # [d][j1 - j0], contiguous (a copy)


def shard_layer(W: torch.Tensor, packed: torch.Tensor, W_down: torch.Tensor, n_m: int, world: int,
                rank: int) -> Shard:
    """This rank's slice of one layer.  W [h][d] and its packed masks are
    sliced by rows without copying (a packed row is d * n_m / 8 bytes, whole
    bytes since d % 8 == 0); W_down [d][h] is sliced by columns into a
    contiguous copy, once, when the layer is loaded."""
    h, d = W.shape
    if W_down.shape != (d, h):
        raise ValueError("W_down must be [d][h]")
    if d % 8:
        raise ValueError("d must be a multiple of 8")
    j0, j1 = shard_range(h, world, rank)
    row_bytes = d * n_m // 8
    return Shard(j0, j1, W[j0:j1], packed[j0 * row_bytes:j1 * row_bytes], W_down[:, j0:j1].contiguous())


def partial(x: torch.Tensor, shard: Shard, n_m: int, act="swish", workspace: Optional[torch.Tensor] = None,
            stream=None) -> torch.Tensor:
    """y_r [T][d]: the FFN block on this rank's hidden units (no exchange)."""
    T, d = x.shape
    if shard.j1 == shard.j0:
        return torch.zeros((T, d), dtype=x.dtype, device=x.device)
    return mglu.forward_down(x, shard.W, shard.packed, n_m, shard.W_down, act, workspace=workspace, stream=stream)


def reduce_partial(y_r: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' partials in place (one all-reduce over the group)."""
    dist.all_reduce(y_r, op=dist.ReduceOp.SUM, group=group)
    return y_r


def ffn_block(x: torch.Tensor, shard: Shard, n_m: int, act="swish", group=None,
              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """y = MGLU(x) W_down^T over the group: the rank's partial, then the all-reduce."""
    return reduce_partial(partial(x, shard, n_m, act, workspace, stream), group)
