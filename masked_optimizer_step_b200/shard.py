"""Row-sharded data-parallel split of the sparse step over several GPUs (host logic).

"Sparse-First Fine-Tuning" (tensorwirelabs.com), section 2.7 splits a step over GPUs by token
positions and exchanges attention keys and values, which needs the forward pass. The split here
stays inside the step itself and shards by rows, which the step allows because every stage is
row-independent once the masks are known:

  * rank g owns a contiguous range of 32-row tiles of every matrix (RowPartition): their q, s,
    delta, live copy and moment slots live on that rank only;
  * each rank holds 1/world of the step's tokens;
  * activity: each rank counts its tokens into the per-row activity (hit counts for the
    embedding, largest |output| for a projection); combine_activity sums the counts and takes the
    largest magnitude across ranks, so every rank then applies the charge rule to the same
    numbers and derives the same masks, lists and slots (the finalize is deterministic);
  * gradients: each rank computes dW = dX^T A (and the embedding-row sums) over its own tokens
    for every globally active row; exchange_rows packs those partial rows by owner and
    reduce-scatters them, so each rank receives the summed gradient of the active rows it owns;
  * update: each rank updates its own active rows.

Collective traffic per step: 4 bytes per row of every matrix (one all-reduce per activity kind)
plus 4*C bytes per active row (one reduce-scatter, each rank receiving its own rows' share).
Everything here is torch.distributed calls and tensor packing; it runs on NCCL for CUDA tensors
and on gloo for CPU tensors.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

TILE = 32


class RowPartition:
    """Contiguous ranges of 32-row tiles of an R-row matrix, one per rank, as even as tiles allow."""

    def __init__(self, R: int, world: int):
        if R % TILE or R <= 0 or world <= 0:
            raise ValueError("R must be a positive multiple of 32 and world positive")
        self.R, self.world = R, world
        tiles = R // TILE
        self.bounds = [TILE * ((tiles * g) // world) for g in range(world + 1)]

    def range(self, rank: int) -> tuple[int, int]:
        return self.bounds[rank], self.bounds[rank + 1]

    def owner(self, rows) -> np.ndarray:
        """Owning rank of each row."""
        return np.searchsorted(np.asarray(self.bounds[1:]), np.asarray(rows), side="right")

    def split(self, rows) -> np.ndarray:
        """For ascending rows, offsets o[0..world] such that rows[o[g]:o[g+1]] are rank g's."""
        return np.searchsorted(np.asarray(rows), np.asarray(self.bounds), side="left")


def combine_activity(hits: torch.Tensor | None = None, magnitudes: torch.Tensor | None = None,
                     group=None):
    """In place across ranks: hit counts are summed, row magnitudes take their largest value.
    Magnitudes may be float32 or the int32 bit patterns of non-negative floats (both order the
    same). Every rank then holds the window's activity over all ranks' tokens."""
    if hits is not None:
        dist.all_reduce(hits, op=dist.ReduceOp.SUM, group=group)
    if magnitudes is not None:
        dist.all_reduce(magnitudes, op=dist.ReduceOp.MAX, group=group)


def exchange_rows(parts, group=None):
    """Sum partial gradient rows over ranks, each rank keeping the rows it owns.

    parts: list, one entry per matrix, of (rows, partial, partition): the matrix's active rows
    (ascending, the same on every rank), this rank's partial gradient of each of them
    ([len(rows) x C], same order) and the matrix's RowPartition. Returns, per matrix, the summed
    gradient of this rank's own active rows ([n_own x C], ascending row order) and those rows.
    One reduce-scatter carries every matrix: each rank's segment holds, matrix after matrix, its
    rows padded to the largest per-rank count of that matrix."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    plan, seg = [], 0
    for rows, partial, part in parts:
        rows = np.asarray(rows)
        assert partial.shape[0] == len(rows) and part.world == world
        off = part.split(rows)
        m = int(np.max(np.diff(off))) if len(rows) else 0
        C = partial.shape[1]
        plan.append((off, m, C, seg))
        seg += m * C
    ref = parts[0][1] if parts else torch.zeros(0)
    send = torch.zeros((world, max(seg, 1)), dtype=ref.dtype, device=ref.device)
    for (rows, partial, part), (off, m, C, base) in zip(parts, plan):
        for g in range(world):
            n = int(off[g + 1] - off[g])
            if n:
                send[g, base:base + n * C] = partial[off[g]:off[g + 1]].reshape(-1)
    recv = torch.empty(max(seg, 1), dtype=ref.dtype, device=ref.device)
    dist.reduce_scatter_tensor(recv, send.reshape(-1), op=dist.ReduceOp.SUM, group=group)
    out = []
    for (rows, partial, part), (off, m, C, base) in zip(parts, plan):
        n = int(off[rank + 1] - off[rank])
        out.append((np.asarray(rows)[off[rank]:off[rank + 1]], recv[base:base + n * C].reshape(n, C)))
    return out
