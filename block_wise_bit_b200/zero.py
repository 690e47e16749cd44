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


class ZeroOneExchange:
    """The collectives of a ZeRO-1 step over one flat parameter list, around the unchanged step.

    Every rank holds the whole flat parameter buffer and its own full gradient (data parallel);
    rank r owns the pieces ``partition(...)[r]``, i.e. one contiguous, block-aligned range of the
    flat buffer (tensors sit at ``offsets`` in it, in list order).  One step is:

      1. ``reduce_scatter_grads``: the gradients are summed over ranks, each rank receiving only
         its own range (ranges are padded to one common chunk length so that the equal-size
         ``reduce_scatter`` collective applies);
      2. the rank steps its pieces with the summed gradient (``piece_views`` gives the slices;
         the optimizer state exists only for the rank's pieces);
      3. ``all_gather_params``: every rank's stepped range is gathered back into every rank's
         flat parameter buffer.

    Works with any torch.distributed backend that has ``reduce_scatter`` and
    ``all_gather_into_tensor`` (NCCL on GPUs, gloo on CPU).  A multi-GPU run is not part of this
    repository's tests (they have one GPU); the exchange is checked with gloo ranks on CPU.
    """

    def __init__(self, numels: Sequence[int], offsets: Sequence[int], blocksize: int, world: int, rank: int,
                 align: int = 16):
        self.world, self.rank, self.blocksize = world, rank, blocksize
        self.numels, self.offsets = list(numels), list(offsets)
        self.pieces = partition(numels, blocksize, world)
        self.ranges = []
        for pcs in self.pieces:
            if pcs:
                lo = self.offsets[pcs[0].tensor] + pcs[0].start
                hi = self.offsets[pcs[-1].tensor] + pcs[-1].start + pcs[-1].numel
            else:
                lo = hi = 0
            self.ranges.append((lo, hi))
        longest = max(hi - lo for lo, hi in self.ranges)
        self.chunk = max(align, (longest + align - 1) // align * align)

    def reduce_scatter_grads(self, g_flat, group=None):
        """Sum of every rank's gradient over this rank's range (a tensor of ``chunk`` elements;
        the first ``hi - lo`` are meaningful)."""
        import torch
        import torch.distributed as dist
        staged = torch.zeros(self.world * self.chunk, dtype=g_flat.dtype, device=g_flat.device)
        for r, (lo, hi) in enumerate(self.ranges):
            staged[r * self.chunk:r * self.chunk + hi - lo].copy_(g_flat[lo:hi])
        out = torch.empty(self.chunk, dtype=g_flat.dtype, device=g_flat.device)
        dist.reduce_scatter(out, list(staged.split(self.chunk)), group=group)
        return out

    def piece_views(self, p_flat, g_chunk):
        """(piece, parameter slice, summed-gradient slice) for each of this rank's pieces."""
        lo = self.ranges[self.rank][0]
        out = []
        for pc in self.pieces[self.rank]:
            a = self.offsets[pc.tensor] + pc.start
            out.append((pc, p_flat[a:a + pc.numel], g_chunk[a - lo:a - lo + pc.numel]))
        return out

    def all_gather_params(self, p_flat, group=None):
        """Copy every rank's range of the flat parameters from that rank into ``p_flat``."""
        import torch
        import torch.distributed as dist
        lo, hi = self.ranges[self.rank]
        mine = torch.zeros(self.chunk, dtype=p_flat.dtype, device=p_flat.device)
        mine[:hi - lo].copy_(p_flat[lo:hi])
        gathered = torch.empty(self.world * self.chunk, dtype=p_flat.dtype, device=p_flat.device)
        dist.all_gather_into_tensor(gathered, mine, group=group)
        for r, (a, b) in enumerate(self.ranges):
            p_flat[a:b].copy_(gathered[r * self.chunk:r * self.chunk + b - a])
