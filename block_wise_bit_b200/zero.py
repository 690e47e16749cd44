"""ZeRO-1 style partition of a tensor list across ranks, on block boundaries.

Blocks are independent (abstract of "8-bit Optimizers via Block-wise Quantization": each block is
quantized on its own and processed in parallel), so the optimizer step shards without any
exchange: split the list's blocks -- numbered tensor by tensor -- into contiguous ranges of
near-equal element count, and let each rank step its range.  A range may cut a tensor, but only
between two of its blocks, so every block (and its absmax) belongs to exactly one rank.
Collectives before and after the step (reduce-scatter of gradients, all-gather of parameters) are
outside the step and outside this module.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

from . import bindings as B


@dataclass(frozen=True)
class Piece:
    tensor: int       # index in the full list
    first_block: int  # first block of the tensor in this piece
    n_blocks: int     # blocks in this piece
    start: int        # first element (first_block * blocksize)
    numel: int        # elements in this piece (the last block of a tensor may be short)


def partition(numels: Sequence[int], blocksize: int, world: int) -> List[List[Piece]]:
    """Contiguous shards of the list's blocks, balanced by element count."""
    if world < 1:
        raise ValueError("world must be >= 1")
    blocks = []  # (tensor, block, elements in block)
    for t, n in enumerate(numels):
        nb = (n + blocksize - 1) // blocksize
        for b in range(nb):
            blocks.append((t, b, min(blocksize, n - b * blocksize)))
    total = sum(x[2] for x in blocks)
    shards: List[List[Piece]] = [[] for _ in range(world)]
    acc, r = 0, 0
    cur = None  # (rank, tensor, first_block, n_blocks, start, numel)

    def flush():
        if cur is not None:
            shards[cur[0]].append(Piece(cur[1], cur[2], cur[3], cur[4], cur[5]))

    for t, b, ne in blocks:
        # move to the next rank once this rank holds its share of the elements
        while r < world - 1 and acc >= (r + 1) * total / world:
            r += 1
        if cur is not None and cur[0] == r and cur[1] == t:
            cur = (r, t, cur[2], cur[3] + 1, cur[4], cur[5] + ne)
        else:
            flush()
            cur = (r, t, b, 1, b * blocksize, ne)
        acc += ne
    flush()
    return shards


def shard_states(states: Sequence[B.TensorState], pieces: Sequence[Piece], blocksize: int) -> List[B.TensorState]:
    """Views of the full list's tensors restricted to one rank's pieces (block-aligned slices;
    the absmax views start at the piece's first block)."""
    out = []
    for pc in pieces:
        ts = states[pc.tensor]
        s, e = pc.start, pc.start + pc.numel
        cut = lambda x: None if x is None else x[s:e]  # noqa: E731
        if ts.absmax1 is not None:
            b0, b1 = pc.first_block, pc.first_block + pc.n_blocks
            cuta = lambda x: None if x is None else x[b0:b1]  # noqa: E731
            out.append(B.TensorState(ts.p[s:e], ts.g[s:e], cut(ts.state1), cut(ts.state2), cuta(ts.absmax1),
                                     cuta(ts.absmax2)))
        else:
            out.append(B.TensorState(ts.p[s:e], ts.g[s:e], cut(ts.state1), cut(ts.state2)))
    return out
