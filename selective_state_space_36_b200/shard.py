"""Partition of one scan workload over the ranks of a multi-GPU job.

The (batch row, channel) pairs of the selective scan are independent SSMs
(NL-345 Mamba translation, section 2 "Structure and Dimensions": the SSM is
applied to every channel separately, B_t and C_t being shared only within a
batch row), so a workload splits over GPUs with no exchange on the data path:
each rank scans its own block of batch rows -- or, when there are fewer rows
than ranks, its own block of channels of every row -- and the gathered
outputs and states are exactly those of one process scanning everything.

Host logic only: no arithmetic of the method lives here.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Shard:
    """Rows [b0, b1) and channels [d0, d1) of the global workload."""
    b0: int
    b1: int
    d0: int
    d1: int

    @property
    def batch(self) -> int:
        return self.b1 - self.b0

    @property
    def dim(self) -> int:
        return self.d1 - self.d0


def _split(n: int, parts: int, i: int, align: int = 1):
    """Part i of [0, n) in `parts` contiguous pieces whose boundaries are
    multiples of `align` (except n itself); sizes differ by at most `align`."""
    units = (n + align - 1) // align
    lo = units * i // parts * align
    hi = units * (i + 1) // parts * align
    return min(lo, n), min(hi, n)


def scan_shard(batch: int, dim: int, world: int, rank: int, channel_align: int = 8) -> Shard:
    """The share of rank `rank` (of `world`) of a (batch, dim) scan workload.

    Batch rows are split when there are at least as many rows as ranks;
    otherwise every row is kept and the channels are split, in multiples of
    `channel_align` so that each rank's rows stay 16-byte aligned for bf16.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if batch >= world:
        b0, b1 = _split(batch, world, rank)
        return Shard(b0, b1, 0, dim)
    d0, d1 = _split(dim, world, rank, channel_align)
    return Shard(0, batch, d0, d1)
