"""Blocks sharded across ranks (shampoo_family_second_b200.sharded), on CPU.

The partition is checked as host logic; the step's communication runs in
real gloo process groups of world size 2, with the float64 oracle standing in
for each rank's block compute (the CUDA optimizer cannot run on CPU ranks).
Every rank must end with the same weights, equal to a single process that
steps all blocks itself.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from shampoo_family_second_b200 import sharded  # noqa: E402

SHAPES = [(96, 80), (40, 70), (64, 64)]
B = 32
HP = dict(beta=0.9, eps=1e-4, lr=1e-2, root_p=4, refresh_every=2)
STEPS = 3


class Cfg:
    block = B


def oracle_local_step(blocks):
    """The float64 oracle over the given blocks, each a parameter of its own."""
    ref = oracle.ShampooOracle([(b[3], b[4]) for b in blocks], B, HP["beta"], HP["eps"], HP["lr"], HP["root_p"],
                               HP["refresh_every"])

    def step(ws, gs):
        P = ref.step([g.numpy() for g in gs])
        for k, w in enumerate(ws):
            w -= torch.from_numpy(HP["lr"] * P[k]).to(w.dtype)
    return step


def gradients(t, rank=None, world=2, shapes=None):
    """Seeded gradients of step t; with a rank, that rank's local part: G plus
    a rank-dependent term whose sum over the ranks is zero (rank 0: +D, rank
    1: -D, any further rank: 0)."""
    shapes = SHAPES if shapes is None else shapes
    rng = np.random.default_rng(100 + t)
    G = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    if rank is None:
        return [torch.from_numpy(g) for g in G]
    D = [np.random.default_rng(200 + t).standard_normal(s).astype(np.float32) for s in shapes]
    sign = {0: 1.0, 1: -1.0}.get(rank, 0.0)
    return [torch.from_numpy(g + np.float32(sign) * d) for g, d in zip(G, D)]


def run_single(grads_reduced, world=2, shapes=None):
    shapes = SHAPES if shapes is None else shapes
    blocks = sharded.block_list(shapes, B)
    opt = sharded.ShardedShampoo(shapes, Cfg, grads_reduced=grads_reduced, local_step=oracle_local_step(blocks))
    W = [torch.zeros(s) for s in shapes]
    for t in range(STEPS):
        if grads_reduced:
            G = gradients(t, shapes=shapes)
        else:  # the average of the ranks' local gradients
            parts = [gradients(t, k, world, shapes) for k in range(world)]
            G = [sum(ps[1:], ps[0]) / world for ps in zip(*parts)]
        opt.step(W, G)
    return [w.numpy().copy() for w in W]


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, grads_reduced, shapes, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        blocks = sharded.block_list(shapes, B)
        owner = sharded.partition_blocks(blocks, world)
        mine = [blocks[i] for i, k in enumerate(owner) if k == rank]
        opt = sharded.ShardedShampoo(shapes, Cfg, grads_reduced=grads_reduced, local_step=oracle_local_step(mine))
        W = [torch.zeros(s) for s in shapes]
        for t in range(STEPS):
            opt.step(W, gradients(t, shapes=shapes) if grads_reduced else gradients(t, rank, world, shapes))
        out_q.put((rank, len(mine), [w.numpy().copy() for w in W]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def run_ranks(grads_reduced, world=2, shapes=None):
    shapes = SHAPES if shapes is None else shapes
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, grads_reduced, shapes, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_block_list_matches_the_oracle_table():
    table = oracle.block_table(SHAPES, B)
    assert sharded.block_list(SHAPES, B) == [(b.param, b.row0, b.col0, b.r, b.c) for b in table]


@pytest.mark.parametrize("world", [1, 2, 3, 8, 40])
def test_partition_covers_and_balances(world):
    blocks = sharded.block_list(SHAPES, B)
    owner = sharded.partition_blocks(blocks, world)
    assert owner == sharded.partition_blocks(blocks, world)  # deterministic
    assert len(owner) == len(blocks) and all(0 <= k < world for k in owner)
    cost = [b[3] ** 3 + b[4] ** 3 for b in blocks]
    load = [sum(c for c, k in zip(cost, owner) if k == r) for r in range(world)]
    # greedy by decreasing cost: no rank exceeds another by more than one block's cost
    assert max(load) - min(load) <= max(cost)
    if world == 1:
        assert set(owner) == {0}


@pytest.mark.parametrize("world", [1, 2, 3])
@pytest.mark.parametrize("grads_reduced", [True, False])
def test_ranks_match_one_process(grads_reduced, world):
    """1 rank (a process group of one: the collective path runs, each
    exchange a copy), 2 ranks (even split) and 3 (uneven segments; the middle
    rank's slice of the gradient reduction): every rank ends with the same
    weights as one process stepping every block.  Sums of three local
    gradients may round differently in the collective, hence a looser bound
    there."""
    single = run_single(grads_reduced, world)
    res = run_ranks(grads_reduced, world)
    counts = [n for _, n, _ in res]
    assert all(n > 0 for n in counts) and sum(counts) == len(sharded.block_list(SHAPES, B))
    tol = 1e-7 if (grads_reduced or world == 2) else 1e-6
    W0 = res[0][2]
    for _, _, W in res[1:]:
        for a, b in zip(W0, W):
            assert np.array_equal(a, b)           # every rank holds the same weights
    for a, s in zip(W0, single):
        assert np.allclose(a, s, rtol=0, atol=tol), float(np.abs(a - s).max())
        assert np.abs(s).max() > 1e-3             # the steps did move the weights


@pytest.mark.parametrize("world", [2, 4, 8])
def test_partition_balance_on_transformer_shapes(world):
    """GPT-2-small layer shapes at block 512 (456 blocks, 252 ragged): the
    busiest rank carries at most 2% more root cost than the average."""
    layer = ((768, 2304), (768, 768), (768, 3072), (3072, 768))
    shapes = [s for _ in range(12) for s in layer]
    blocks = sharded.block_list(shapes, 512)
    assert len(blocks) == 456
    owner = sharded.partition_blocks(blocks, world)
    cost = [b[3] ** 3 + b[4] ** 3 for b in blocks]
    load = [sum(c for c, k in zip(cost, owner) if k == r) for r in range(world)]
    assert max(load) <= 1.02 * sum(load) / world, load


@pytest.mark.parametrize("grads_reduced", [True, False])
def test_more_ranks_than_blocks(grads_reduced):
    """A 40 x 30 weight at block 32 has 2 blocks; with 3 ranks one rank owns
    none.  It still takes part in every collective, and all ranks end with
    the single-process weights."""
    shapes = [(40, 30)]
    single = run_single(grads_reduced, 3, shapes)
    res = run_ranks(grads_reduced, 3, shapes)
    assert sorted(n for _, n, _ in res) == [0, 1, 1]
    for _, _, W in res:
        for a, s_ in zip(W, single):
            assert np.allclose(a, s_, rtol=0, atol=1e-6), float(np.abs(a - s_).max())


def test_partition_properties_on_random_shapes():
    """Random weight lists, block sizes and world sizes: the blocks tile every
    weight exactly once, every block has one owner, and the greedy balance
    bound holds (no rank carries more than the average plus one block's cost)."""
    hypothesis = pytest.importorskip("hypothesis")
    st = hypothesis.strategies

    @hypothesis.settings(max_examples=60, deadline=None)
    @hypothesis.given(shapes=st.lists(st.tuples(st.integers(1, 300), st.integers(1, 300)), min_size=1, max_size=6),
                      block=st.sampled_from([32, 64, 128]), world=st.integers(1, 9))
    def check(shapes, block, world):
        blocks = sharded.block_list(shapes, block)
        for p, (m, n) in enumerate(shapes):
            cover = np.zeros((m, n), dtype=int)
            for q, r0, c0, r, c in blocks:
                if q == p:
                    assert 0 < r <= block and 0 < c <= block
                    cover[r0:r0 + r, c0:c0 + c] += 1
            assert (cover == 1).all()
        owner = sharded.partition_blocks(blocks, world)
        assert len(owner) == len(blocks) and all(0 <= k < world for k in owner)
        cost = [b[3] ** 3 + b[4] ** 3 for b in blocks]
        load = [sum(c for c, k in zip(cost, owner) if k == r) for r in range(world)]
        assert max(load) <= sum(load) / world + max(cost)

    check()


class FakeComm:
    """In-process collectives for ranks run as threads: the reduce-scatter and
    all-gather semantics of NCCL's reduce_scatter_tensor /
    all_gather_into_tensor on flat tensors."""

    def __init__(self, world):
        import threading
        self.world = world
        self.bar = threading.Barrier(world)
        self.slots = [None] * world

    def reduce_scatter(self, rank):
        def rs(out, inp):
            self.slots[rank] = inp.clone()
            self.bar.wait()
            n = out.numel()
            out.copy_(sum(s[rank * n:(rank + 1) * n] for s in self.slots))
            self.bar.wait()
        return rs

    def all_gather(self, rank):
        def ag(out, inp):
            self.slots[rank] = inp.clone()
            self.bar.wait()
            out.copy_(torch.cat(self.slots))
            self.bar.wait()
        return ag


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("grads_reduced", [True, False])
def test_injected_collectives_match_one_process(grads_reduced, world):
    """The reduce-scatter / all-gather branch (the one NCCL takes) with its
    packing and segment offsets, run with in-process collectives: every rank
    (a thread) ends with the single-process weights."""
    import threading
    comm = FakeComm(world)
    blocks = sharded.block_list(SHAPES, B)
    owner = sharded.partition_blocks(blocks, world)
    results = [None] * world
    errors = []

    def rank_main(rank):
        try:
            mine = [blocks[i] for i, k in enumerate(owner) if k == rank]
            opt = sharded.ShardedShampoo(SHAPES, Cfg, grads_reduced=grads_reduced,
                                         local_step=oracle_local_step(mine), world=world, rank=rank,
                                         reduce_scatter=comm.reduce_scatter(rank), all_gather=comm.all_gather(rank))
            W = [torch.zeros(s) for s in SHAPES]
            for t in range(STEPS):
                opt.step(W, gradients(t, shapes=SHAPES) if grads_reduced else gradients(t, rank, world))
            results[rank] = [w.numpy().copy() for w in W]
        except Exception as e:   # surfaced below
            errors.append(e)
            comm.bar.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(world)]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=120)
    assert not errors, errors
    single = run_single(grads_reduced, world)
    tol = 1e-7 if (grads_reduced or world == 2) else 1e-6
    for W in results[1:]:
        for a, b in zip(results[0], W):
            assert np.array_equal(a, b)
    for a, s in zip(results[0], single):
        assert np.allclose(a, s, rtol=0, atol=tol), float(np.abs(a - s).max())


def test_packed_offsets_tile_each_segment():
    """Every block's packed range lies inside its owner's segment and the
    ranges of one segment do not overlap."""
    blocks = sharded.block_list(SHAPES, B)
    for world in (1, 2, 3, 5):
        owner = sharded.partition_blocks(blocks, world)
        segments, offsets, seg = sharded.packed_offsets(blocks, owner, world)
        for rank, sg in enumerate(segments):
            used = np.zeros(seg, dtype=int)
            for i in sg:
                n = blocks[i][3] * blocks[i][4]
                assert 0 <= offsets[i] and offsets[i] + n <= seg
                used[offsets[i]:offsets[i] + n] += 1
            assert used.max(initial=0) <= 1
