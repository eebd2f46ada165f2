"""Blocked Shampoo with its blocks sharded across data-parallel ranks.

The blocks of the blocked step are independent units: each owns its L, R and
roots.  So each rank keeps the statistics and roots of the blocks assigned to
it, updates only those blocks' weights, and the updated blocks are then
all-gathered so that every rank holds the full weights (DASH abstract: the
preconditioner blocks are distributed across devices; Distributed Shampoo
likewise assigns blocks to workers).

Partition: whole blocks, balanced by the root cost r^3 + c^3 of a block
(longest-processing-time greedy, ties to the lower rank), which is the
O(m^3 + n^3) term that dominates the step.

Gradients:
  * ``grads_reduced=True`` (default): the caller passes gradients already
    averaged over ranks (the usual data-parallel all-reduce).  Each rank steps
    its blocks in place through strided views of the full weights.
  * ``grads_reduced=False``: the caller passes each rank's local gradients;
    they are summed by block owner (a reduce-scatter, or an all-reduce where the
    backend has no reduce-scatter) and divided by the world size.

Communication uses torch.distributed (NCCL on GPUs); every step runs the same
collectives in the same order on all ranks.  ``local_step`` replaces the
blocks' compute (the CUDA optimizer by default) so that the communication can
be exercised on CPU ranks.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

Block = Tuple[int, int, int, int, int]  # (param, row0, col0, r, c)


def block_list(shapes: Sequence[Tuple[int, int]], block: int) -> List[Block]:
    """Every B x B block of every weight, in (param, block row, block column)
    order; the last row / column of blocks keeps its real size."""
    out = []
    for p, (m, n) in enumerate(shapes):
        for r0 in range(0, m, block):
            for c0 in range(0, n, block):
                out.append((p, r0, c0, min(block, m - r0), min(block, n - c0)))
    return out


def partition_blocks(blocks: Sequence[Block], world: int) -> List[int]:
    """Owner rank of each block: blocks in decreasing root cost r^3 + c^3 (ties
    by index) go to the rank with the least cost so far (ties to the lower
    rank)."""
    if world < 1:
        raise ValueError("world size must be >= 1")
    order = sorted(range(len(blocks)), key=lambda i: (-(blocks[i][3] ** 3 + blocks[i][4] ** 3), i))
    load = [0] * world
    owner = [0] * len(blocks)
    for i in order:
        k = min(range(world), key=lambda j: (load[j], j))
        owner[i] = k
        load[k] += blocks[i][3] ** 3 + blocks[i][4] ** 3
    return owner


class ShardedShampoo:
    """Blocked Shampoo over a list of 2-D weights, blocks sharded across the
    ranks of ``group`` (the default process group, or a single process when
    torch.distributed is not initialised)."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], cfg, group=None, grads_reduced: bool = True,
                 local_step: Optional[Callable] = None, device=None):
        import torch
        import torch.distributed as dist

        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.block = int(cfg.block)
        self.group = group
        self.distributed = dist.is_available() and dist.is_initialized()
        self.rank = dist.get_rank(group) if self.distributed else 0
        self.world = dist.get_world_size(group) if self.distributed else 1
        self.grads_reduced = grads_reduced
        self.blocks = block_list(self.shapes, self.block)
        self.owner = partition_blocks(self.blocks, self.world)
        self.owned = [i for i, k in enumerate(self.owner) if k == self.rank]
        # each rank's blocks, in block order, packed back to back
        self.segments = [[i for i, k in enumerate(self.owner) if k == rank] for rank in range(self.world)]
        sizes = [sum(self.blocks[i][3] * self.blocks[i][4] for i in seg) for seg in self.segments]
        self.seg_elems = max(sizes) if sizes else 0
        self.device = torch.device(device) if device is not None else None
        if local_step is None:
            from . import Shampoo
            opt = Shampoo([(self.blocks[i][3], self.blocks[i][4]) for i in self.owned], cfg,
                          device=self.device) if self.owned else None
            local_step = (lambda ws, gs: opt.step(ws, gs)) if opt is not None else (lambda ws, gs: None)
            self.local_optimizer = opt
        self.local_step = local_step

    # -- helpers -------------------------------------------------------------
    def _view(self, t, i):
        p, r0, c0, r, c = self.blocks[i]
        return t[r0:r0 + r, c0:c0 + c]

    def _pack(self, tensors, seg, out):
        o = 0
        for i in seg:
            v = self._view(tensors[self.blocks[i][0]], i)
            n = v.numel()
            out[o:o + n].copy_(v.reshape(-1))
            o += n
        return out

    def _unpack(self, buf, seg, tensors):
        o = 0
        for i in seg:
            v = self._view(tensors[self.blocks[i][0]], i)
            n = v.numel()
            v.copy_(buf[o:o + n].view(v.shape))
            o += n

    def _backend(self):
        import torch.distributed as dist
        return dist.get_backend(self.group) if self.distributed else None

    # -- the step ------------------------------------------------------------
    def step(self, weights, grads):
        """One sharded step.  ``weights``: this rank's full fp32 weights
        (updated in place; equal on every rank afterwards).  ``grads``: full
        gradients, averaged over ranks or local (see the class)."""
        import torch
        import torch.distributed as dist

        if len(weights) != len(self.shapes) or len(grads) != len(self.shapes):
            raise ValueError("one weight and one gradient per shape")
        dev = weights[0].device
        mine = self.segments[self.rank]
        if self.grads_reduced:
            self.local_step([self._view(weights[self.blocks[i][0]], i) for i in mine],
                            [self._view(grads[self.blocks[i][0]], i) for i in mine])
        else:
            # sum the local gradients by block owner, in fp32 (also for bf16 gradients)
            gbuf = torch.zeros(self.world * self.seg_elems, dtype=torch.float32, device=dev)
            for rank, seg in enumerate(self.segments):
                self._pack(grads, seg, gbuf[rank * self.seg_elems:(rank + 1) * self.seg_elems])
            if self.world > 1:
                if self._backend() == "nccl":
                    out = torch.empty(self.seg_elems, dtype=gbuf.dtype, device=dev)
                    dist.reduce_scatter_tensor(out, gbuf, group=self.group)
                else:  # no reduce-scatter on this backend: all-reduce and keep this rank's part
                    dist.all_reduce(gbuf, group=self.group)
                    out = gbuf[self.rank * self.seg_elems:(self.rank + 1) * self.seg_elems]
            else:
                out = gbuf
            gmine = (out / self.world).to(grads[0].dtype)
            wmine = self._pack(weights, mine, torch.empty(self.seg_elems, dtype=weights[0].dtype, device=dev))
            ws, gs, o = [], [], 0
            for i in mine:
                r, c = self.blocks[i][3], self.blocks[i][4]
                ws.append(wmine[o:o + r * c].view(r, c))
                gs.append(gmine[o:o + r * c].view(r, c))
                o += r * c
            self.local_step(ws, gs)
            self._unpack(wmine, mine, weights)
        if self.world > 1:
            wbuf = torch.zeros(self.seg_elems, dtype=weights[0].dtype, device=dev)
            self._pack(weights, mine, wbuf)
            parts = [torch.empty_like(wbuf) for _ in range(self.world)]
            dist.all_gather(parts, wbuf, group=self.group)
            for rank, seg in enumerate(self.segments):
                if rank != self.rank:
                    self._unpack(parts[rank], seg, weights)
