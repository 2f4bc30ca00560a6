"""Splitting a tensor's groups across ranks (one process per GPU).

Every 512-bit block is self-contained and the tables are per tensor, so the
codec shards with no exchange: each rank encodes or decodes a contiguous range
of rows of the group descriptor, and nothing crosses between ranks on the data
path.  These helpers compute that range and the descriptor of a rank's share.
"""
from __future__ import annotations

from ._lib import Desc


def shard_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of rank's share of n items, as equal as possible."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard arguments")
    return n * rank // world, n * (rank + 1) // world


def shard_desc(d: Desc, rank: int, world: int) -> Desc:
    """The rows of descriptor d that belong to `rank`; a single-row descriptor
    is split along its groups instead."""
    if d.rows > 1 or d.groups_per_row == 0:
        a, b = shard_range(d.rows, rank, world)
        return Desc(b - a, d.groups_per_row, d.src_row_stride, d.dst_row_stride,
                    d.src_offset + a * d.src_row_stride, d.dst_offset + a * d.dst_row_stride)
    a, b = shard_range(d.groups_per_row, rank, world)
    return Desc(1 if b > a else 0, b - a, d.src_row_stride, d.dst_row_stride,
                d.src_offset + a, d.dst_offset + a)


def whole_job_rate(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job throughput: units of all ranks over the slowest rank's time."""
    return units_per_rank * world / (max_ms * 1e-3)
