"""Row sharding of an OWQ layer over the ranks of a process group (host logic).

The output rows of the product are independent ("Error Decomposition" on the paperlayer.ai
summary of the OWQ paper: a row's quantisation error involves no other row), so a layer splits
by output rows with no reduction: each rank packs its own contiguous block of rows -- whole
16-row tiles, the decode kernel's unit -- runs the product on them, and the ranks all-gather
the M x N output.  The weak-column index list and the activations are replicated.

This module is argument bookkeeping only: which rows a rank owns, the slices of the quantised
operands that go to owq_pack, and the all-gather that reassembles y in row order.  Every
product runs in the CUDA library.
"""
from __future__ import annotations

TILE = 16   # rows of the decode kernel's tile: shards are whole tiles, the last one ragged


def row_range(N: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [lo, hi) of `rank`: tiles dealt as evenly as possible, lower ranks first."""
    if world < 1 or not 0 <= rank < world or N < 1:
        raise ValueError("bad world/rank/N")
    tiles = (N + TILE - 1) // TILE
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(N, t0 * TILE), min(N, t1 * TILE)


def shard_operands(q: dict, lo: int, hi: int) -> dict:
    """The row slices [lo, hi) of quantised operands (codes, scales, zeros, w_weak: row-major
    N x ...); idx is shared by every rank.  Works on numpy arrays and torch tensors."""
    out = {key: q[key][lo:hi] for key in ("codes", "scales", "zeros", "w_weak") if key in q}
    out["idx"] = q["idx"]
    return out


def all_gather_rows(y_local, N: int, world: int, group=None):
    """Reassemble y (M x N) from the ranks' M x (hi - lo) blocks, in row order.  Blocks are
    padded to the largest shard for the collective and cut back after it."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return y_local
    M = y_local.shape[0]
    sizes = [row_range(N, world, r) for r in range(world)]
    width = max(hi - lo for lo, hi in sizes)
    pad = torch.zeros((M, width), dtype=y_local.dtype, device=y_local.device)
    pad[:, : y_local.shape[1]] = y_local
    bufs = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(bufs, pad.contiguous(), group=group)
    return torch.cat([b[:, : hi - lo] for b, (lo, hi) in zip(bufs, sizes)], dim=1)
