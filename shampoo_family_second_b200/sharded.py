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
  * ``grads_reduced=False``: the caller passes each rank's local gradients.
    They are packed by block owner, each scaled by 1/world (fp32, also for
    bf16 gradients, which are widened exactly), and summed by a reduce-scatter
    (or an all-reduce plus slice where the backend has no reduce-scatter): each
    rank receives the average of its own blocks' gradients in fp32, and steps
    its blocks on that (its local optimizer takes fp32 gradients).

Packed layout: the blocks of rank k lie in segment k of a buffer of
world x seg_elems floats, in block order, each row-major r x c.  On CUDA
tensors one kernel launch (shampoo_pack_blocks) gathers or scatters a whole
block list; buffers are allocated once.

Communication uses torch.distributed (NCCL on GPUs); every step runs the same
collectives in the same order on all ranks.  Whenever a process group is
initialised (or collectives are injected) the collective path runs, also with
a single rank, where the exchange is a copy; only a single process without a
group skips it.  ``reduce_scatter(out, inp)`` and
``all_gather(out, inp)`` (flat tensors: out = the rank's segment of the sum
of inp over ranks; out = every rank's inp, back to back) may be injected to
replace them, and ``local_step`` replaces the blocks' compute (the CUDA
optimizer by default), so that the packing, offsets and collectives can be
exercised on CPU.
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


def packed_offsets(blocks: Sequence[Block], owner: Sequence[int], world: int):
    """(segments, offsets, seg_elems): the blocks of each rank in block order,
    each block's first float within its owner's segment, and the segment
    length (the largest rank's total, so that every segment has one size)."""
    segments = [[i for i, k in enumerate(owner) if k == rank] for rank in range(world)]
    offsets = [0] * len(blocks)
    sizes = []
    for seg in segments:
        o = 0
        for i in seg:
            offsets[i] = o
            o += blocks[i][3] * blocks[i][4]
        sizes.append(o)
    return segments, offsets, max(sizes) if sizes else 0


class ShardedShampoo:
    """Blocked Shampoo over a list of 2-D weights, blocks sharded across the
    ranks of ``group`` (the default process group, or a single process when
    torch.distributed is not initialised)."""

    def __init__(self, shapes: Sequence[Tuple[int, int]], cfg, group=None, grads_reduced: bool = True,
                 local_step: Optional[Callable] = None, device=None, world: Optional[int] = None,
                 rank: Optional[int] = None, reduce_scatter: Optional[Callable] = None,
                 all_gather: Optional[Callable] = None):
        import torch
        import torch.distributed as dist

        self.shapes = [tuple(int(x) for x in s) for s in shapes]
        self.block = int(cfg.block)
        self.group = group
        self.distributed = dist.is_available() and dist.is_initialized()
        self.rank = rank if rank is not None else (dist.get_rank(group) if self.distributed else 0)
        self.world = world if world is not None else (dist.get_world_size(group) if self.distributed else 1)
        self.grads_reduced = grads_reduced
        self.blocks = block_list(self.shapes, self.block)
        self.owner = partition_blocks(self.blocks, self.world)
        self.owned = [i for i, k in enumerate(self.owner) if k == self.rank]
        self.segments, self.offsets, self.seg_elems = packed_offsets(self.blocks, self.owner, self.world)
        self.device = torch.device(device) if device is not None else None
        self._rs = reduce_scatter if reduce_scatter is not None else self._default_reduce_scatter
        self._ag = all_gather if all_gather is not None else self._default_all_gather
        self.collective = self.world > 1 or self.distributed or reduce_scatter is not None or all_gather is not None
        self._bufs = None
        self._packers = None
        self.local_optimizer = None
        if local_step is None:
            from . import F32, Shampoo
            local_cfg = cfg
            if not grads_reduced and getattr(cfg, "grad_dtype", F32) != F32:
                import copy
                local_cfg = copy.copy(cfg)     # averaged gradients arrive as fp32
                local_cfg.grad_dtype = F32
            opt = Shampoo([(self.blocks[i][3], self.blocks[i][4]) for i in self.owned], local_cfg,
                          device=self.device) if self.owned else None
            local_step = (lambda ws, gs: opt.step(ws, gs)) if opt is not None else (lambda ws, gs: None)
            self.local_optimizer = opt
        self.local_step = local_step

    # -- collectives ---------------------------------------------------------
    def _backend(self):
        import torch.distributed as dist
        return dist.get_backend(self.group) if self.distributed else None

    def _default_reduce_scatter(self, out, inp):
        import torch.distributed as dist
        if self._backend() == "nccl":
            dist.reduce_scatter_tensor(out, inp, group=self.group)
        else:  # no reduce-scatter on this backend: all-reduce and keep this rank's part
            dist.all_reduce(inp, group=self.group)
            out.copy_(inp[self.rank * self.seg_elems:(self.rank + 1) * self.seg_elems])

    def _default_all_gather(self, out, inp):
        import torch.distributed as dist
        if self._backend() == "nccl":
            dist.all_gather_into_tensor(out, inp, group=self.group)
        else:
            dist.all_gather(list(out.view(self.world, -1).unbind(0)), inp, group=self.group)

    # -- packing -------------------------------------------------------------
    def _view(self, t, i):
        p, r0, c0, r, c = self.blocks[i]
        return t[r0:r0 + r, c0:c0 + c]

    def _ensure(self, dev):
        import torch
        if self._bufs is not None:
            return
        n = self.seg_elems
        f32 = dict(dtype=torch.float32, device=dev)
        self._bufs = {"gall": torch.zeros(max(self.world * n, 1), **f32), "gmine": torch.zeros(max(n, 1), **f32),
                      "wmine": torch.zeros(max(n, 1), **f32), "wall": torch.zeros(max(self.world * n, 1), **f32)}
        if dev.type == "cuda":
            from . import BlockPacker
            every = [b + (self.owner[i] * n + self.offsets[i],) for i, b in enumerate(self.blocks)]
            own = [self.blocks[i] + (self.offsets[i],) for i in self.owned]
            self._packers = {"all": BlockPacker(every, dev), "own": BlockPacker(own, dev)}

    def _gather(self, which, mats, out, scale=1.0):
        if self._packers is not None:
            self._packers[which].gather(mats, out, scale)
            return
        blocks = range(len(self.blocks)) if which == "all" else self.owned
        for i in blocks:
            base = (self.owner[i] * self.seg_elems if which == "all" else 0) + self.offsets[i]
            v = self._view(mats[self.blocks[i][0]], i)
            out[base:base + v.numel()].copy_(v.reshape(-1).to(out.dtype) * scale if scale != 1.0
                                             else v.reshape(-1).to(out.dtype))

    def _scatter(self, which, buf, mats):
        if self._packers is not None:
            self._packers[which].scatter(buf, mats)
            return
        blocks = range(len(self.blocks)) if which == "all" else self.owned
        for i in blocks:
            base = (self.owner[i] * self.seg_elems if which == "all" else 0) + self.offsets[i]
            v = self._view(mats[self.blocks[i][0]], i)
            v.copy_(buf[base:base + v.numel()].view(v.shape))

    def _own_views(self, buf):
        out = []
        for i in self.owned:
            r, c = self.blocks[i][3], self.blocks[i][4]
            o = self.offsets[i]
            out.append(buf[o:o + r * c].view(r, c))
        return out

    # -- the step ------------------------------------------------------------
    def step(self, weights, grads):
        """One sharded step.  ``weights``: this rank's full fp32 weights
        (updated in place; equal on every rank afterwards).  ``grads``: full
        gradients, averaged over ranks or local (see the class)."""
        if len(weights) != len(self.shapes) or len(grads) != len(self.shapes):
            raise ValueError("one weight and one gradient per shape")
        dev = weights[0].device
        self._ensure(dev)
        b = self._bufs
        n = self.seg_elems
        if self.grads_reduced:
            self.local_step([self._view(weights[self.blocks[i][0]], i) for i in self.owned],
                            [self._view(grads[self.blocks[i][0]], i) for i in self.owned])
            if self.collective:
                self._gather("own", weights, b["wmine"][:n])
        else:
            gall = b["gall"][:self.world * n]
            self._gather("all", grads, gall, 1.0 / self.world)
            gmine = b["gmine"][:n]
            if self.collective:
                self._rs(gmine, gall)
            else:
                gmine.copy_(gall)
            self._gather("own", weights, b["wmine"][:n])
            self.local_step(self._own_views(b["wmine"]), self._own_views(gmine))
            if not self.collective:
                self._scatter("own", b["wmine"], weights)
        if self.collective:
            wall = b["wall"][:self.world * n]
            self._ag(wall, b["wmine"][:n])
            self._scatter("all", wall, weights)
