"""ZeRO-1 style partition of a tensor list across ranks, on block boundaries.

Blocks are independent (abstract of "8-bit Optimizers via Block-wise Quantization": each block is
quantized on its own and processed in parallel), so the optimizer step shards without any
exchange: each rank steps one contiguous range of the list's blocks.  A range may cut a tensor,
but only between two of its blocks, so every block (and its absmax) belongs to exactly one rank.
The collectives of a data-parallel step -- reduce-scatter of gradients before the step,
all-gather of parameters after it -- are outside the step kernel (``ZeroOneExchange``).
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

    Flat layout: tensor i occupies ``[offsets[i], offsets[i] + numels[i])`` of a flat buffer whose
    offsets are multiples of the blocksize, so every offset that is a multiple of the blocksize is
    a block boundary of whatever tensor it falls in.  The buffer is ``world * chunk`` elements
    long (``chunk`` a multiple of the blocksize, the tail is padding) and rank r owns
    ``[r * chunk, (r + 1) * chunk)``: an equal, block-aligned share.  Every rank holds the whole
    flat parameter buffer and its own full gradient (data parallel).  One step is:

      1. ``reduce_scatter_grads``: the gradients are summed over ranks into this rank's range of
         its own gradient buffer, in place (``reduce_scatter_tensor`` on the flat buffer);
      2. the rank steps its pieces with the summed gradient (``piece_views``; the optimizer state
         exists only for the rank's pieces);
      3. ``all_gather_params``: every rank's stepped range is gathered into every rank's flat
         parameter buffer, in place (``all_gather_into_tensor``).

    No staging copies: both collectives read and write the flat buffers directly.  Works with any
    torch.distributed backend that has ``reduce_scatter_tensor`` and ``all_gather_into_tensor``
    (NCCL on GPUs, gloo on CPU).
    """

    def __init__(self, numels: Sequence[int], blocksize: int, world: int, rank: int):
        if world < 1 or not 0 <= rank < world:
            raise ValueError("need 0 <= rank < world")
        self.world, self.rank, self.blocksize = world, rank, blocksize
        self.numels = list(numels)
        self.offsets, o = [], 0
        for n in self.numels:
            self.offsets.append(o)
            o += (n + blocksize - 1) // blocksize * blocksize
        blocks = o // blocksize
        self.chunk = max(1, (blocks + world - 1) // world) * blocksize
        self.total = world * self.chunk
        self.pieces = [self._pieces(r) for r in range(world)]

    @property
    def range(self):
        """This rank's range of the flat buffers."""
        return self.rank * self.chunk, (self.rank + 1) * self.chunk

    def _pieces(self, r: int) -> List[Piece]:
        lo, hi = r * self.chunk, (r + 1) * self.chunk
        out = []
        for t, (n, off) in enumerate(zip(self.numels, self.offsets)):
            a, b = max(lo, off), min(hi, off + n)
            if a >= b:
                continue
            s, e = a - off, b - off  # s is a multiple of the blocksize (block boundary)
            nb = (e - s + self.blocksize - 1) // self.blocksize
            out.append(Piece(t, s // self.blocksize, nb, s, e - s))
        return out

    def views(self, flat, t: int):
        """Tensor t's slice of a flat buffer."""
        return flat[self.offsets[t]:self.offsets[t] + self.numels[t]]

    def reduce_scatter_grads(self, g_flat, group=None):
        """Sum every rank's gradient over this rank's range, written into ``g_flat`` in place;
        returns that range (a view)."""
        import torch.distributed as dist
        lo, hi = self.range
        out = g_flat[lo:hi]
        dist.reduce_scatter_tensor(out, g_flat[:self.total], group=group)
        return out

    def piece_views(self, p_flat, g_flat):
        """(piece, parameter slice, gradient slice) for each of this rank's pieces."""
        out = []
        for pc in self.pieces[self.rank]:
            a = self.offsets[pc.tensor] + pc.start
            out.append((pc, p_flat[a:a + pc.numel], g_flat[a:a + pc.numel]))
        return out

    def all_gather_params(self, p_flat, group=None):
        """Every rank's range of the flat parameters, from that rank into ``p_flat``, in place."""
        import torch.distributed as dist
        lo, hi = self.range
        dist.all_gather_into_tensor(p_flat[:self.total], p_flat[lo:hi], group=group)
