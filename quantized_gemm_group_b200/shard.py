"""Splitting one weight-only linear layer over the GPUs of a node by output
channels, and gathering its output.

The layer y = x . dequant(W)^T shards along N (the output channels) with no
exchange before the product: every rank holds whole 128-row blocks of W (the
block is the unit of the interleaved layout and of a Layer-mix / Channel-mix
width map, so a rank's rows are a contiguous slice of the packed codes, scales
and zeros), computes y for its rows, and one all-gather assembles y.  Splitting
K instead would need an all-reduce of fp32 partial sums, which moves more
bytes.  Host logic only; the product on each rank is bq_linear.
"""
from __future__ import annotations

import numpy as np
import torch

from . import bq

BLOCK = 128


def block_ranges(N: int, world: int, bit_map=None) -> list[tuple[int, int]]:
    """Contiguous row ranges [r0, r1), one per rank, made of whole 128-row
    blocks (a last partial block of N % 128 rows stays whole).  Ranks get
    blocks in order and as equal a share of the blocks' packed bytes as whole
    blocks allow: every block counts the same at a uniform width (a short
    last block included), a 4-bit block twice a 2-bit one under a width map.
    A rank gets no rows when there are fewer blocks than ranks."""
    if N < 0 or world < 1:
        raise ValueError("N >= 0 and world >= 1 required")
    nblk = (N + BLOCK - 1) // BLOCK
    if bit_map is not None:
        w = np.asarray(bit_map, dtype=np.float64)
        if len(w) != nblk:
            raise ValueError("bit map needs one entry per 128-row block")
    else:
        w = np.ones(nblk)
    cum = np.concatenate([[0.0], np.cumsum(w)])
    total = cum[-1]
    cuts = [0]
    for r in range(1, world):
        # first block boundary whose prefix reaches r/world of the bytes
        b = int(np.searchsorted(cum, total * r / world - 1e-9, side="left"))
        b = min(max(b, cuts[-1]), nblk)
        # take the nearer boundary (b - 1 or b) to the target
        if b > cuts[-1] and abs(cum[b - 1] - total * r / world) < abs(cum[b] - total * r / world):
            b -= 1
        cuts.append(b)
    cuts.append(nblk)
    return [(min(cuts[i] * BLOCK, N), min(cuts[i + 1] * BLOCK, N)) for i in range(world)]


def gather_rows(y_local: torch.Tensor, ranges, rank: int, group=None) -> torch.Tensor:
    """All-gather the ranks' [M, r1 - r0] outputs into y [M, N] (slices padded
    to the largest one for the collective, then trimmed)."""
    import torch.distributed as dist
    world = len(ranges)
    M = y_local.shape[0]
    width = max(r1 - r0 for r0, r1 in ranges)
    pad = torch.zeros((width, M), dtype=y_local.dtype, device=y_local.device)
    mine = ranges[rank][1] - ranges[rank][0]
    if mine:
        pad[:mine] = y_local.t()
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad.contiguous(), group=group)
    cols = [parts[i][:r1 - r0] for i, (r0, r1) in enumerate(ranges)]
    return torch.cat(cols, dim=0).t().contiguous()


class ShardedLinear:
    """This rank's rows of one weight-only linear (uniform width): quantized
    on the device by bq_quantize into the interleaved layout, y gathered from
    every rank."""

    def __init__(self, W: torch.Tensor, bits: int, group: int, rank: int, world: int):
        self.N, self.K = W.shape
        self.bits, self.group = bits, group
        self.ranges = block_ranges(self.N, world)
        self.rank = rank
        r0, r1 = self.ranges[rank]
        self.rows = r1 - r0
        self.q = bq.bq_quantize(W[r0:r1].contiguous(), bits, group, "interleaved") if self.rows else None

    def local(self, x: torch.Tensor, out=None, stream=None) -> torch.Tensor:
        if not self.rows:
            return torch.empty((x.shape[0], 0), dtype=x.dtype, device=x.device)
        pk, sc, ze = self.q
        return bq.bq_linear(x, pk, sc, ze, self.rows, self.bits, self.group, out=out, stream=stream)

    def __call__(self, x: torch.Tensor, group=None) -> torch.Tensor:
        return gather_rows(self.local(x), self.ranges, self.rank, group)
