"""Host logic of multi-GPU runs, on CPU with the gloo backend (world size 2).

Blocks are independent (each has its own L and R), so several GPUs run
weak-scaled replicas of the step with no exchange on the data path.  What
multi-rank runs add is host logic: per-rank seeding, the maximum of the
timings over ranks, the whole-job rate, and rank 0 alone printing.  These
tests drive that logic through real gloo process groups.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        r, w, _ = bench.dist_env()
        # per-rank step and e2e timings; rank 1 is the slower in the first, rank 0 in the second
        mine = [10.0 + 5.0 * r, 30.0 - 3.0 * r]
        total, e2e = bench.max_over_ranks(mine, w, "cpu")
        rate = bench.job_throughput(128, w, total)
        # each rank draws its own gradients (seed offset by rank) with the workload's recipe
        wl = workloads.workload("lowrank")
        g = bench.device_gradients(wl, wl.seed + 1000 * r, 1, "cpu")[0][0]
        gathered = [torch.zeros_like(g) for _ in range(w)]
        dist.all_gather(gathered, g)
        same = bool(torch.equal(gathered[0], gathered[1]))
        out_q.put((r, total, e2e, rate, same, tuple(g.shape), float(g.std())))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def two_rank_results():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_timing_is_max_over_ranks(two_rank_results):
    for _, total, e2e, _, _, _, _ in two_rank_results:
        assert total == 15.0      # rank 1's step time
        assert e2e == 30.0        # rank 0's end-to-end time


def test_weak_scaled_rate_counts_every_rank(two_rank_results):
    for _, total, _, rate, _, _, _ in two_rank_results:
        assert rate == pytest.approx(128 * 2 / (total * 1e-3))
        # both ranks report the same job-wide number
    assert two_rank_results[0][3] == two_rank_results[1][3]


def test_replicas_draw_different_gradients_of_the_same_recipe(two_rank_results):
    (_, _, _, _, same0, shape0, sd0), (_, _, _, _, same1, shape1, sd1) = two_rank_results
    assert not same0 and not same1
    assert shape0 == shape1 == (1024, 1024)
    # low rank (unit entry variance) plus noise: both ranks near 1
    assert 0.5 < sd0 < 2.0 and 0.5 < sd1 < 2.0


def test_single_rank_helpers():
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
    assert bench.job_throughput(10, 1, 0.0) == 0.0
    assert bench.job_throughput(10, 4, 1000.0) == pytest.approx(40.0)


def test_reference_arm_only_rank0_prints():
    """Under torchrun the reference arm runs on rank 0 alone; other ranks exit
    0 without work (and without output)."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_line_rank0():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "3", "--cpu-budget-s", "2"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["unit"] == "inverse-roots/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["higher_is_better"] is True and line["steps"] == 2 and line["warmup"] == 3
