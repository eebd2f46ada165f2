"""Benchmark of the blocked Shampoo step on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path (stack -> statistics -> inverse roots
when the step is a refresh step -> apply + update) over one batch of synthetic
gradients, through the C ABI (libshampoo.so).  Default workload: Llama-1B layer
shapes (16 layers x {4 x 2048x2048, 2 x 2048x8192, 8192x2048}), block 1024
(1024 blocks -> 2048 roots per refresh), bf16 gradients N(0, 0.01^2), fp32
statistics and roots, beta 0.999, eps 1e-10, roots refreshed every 10 steps:
the largest single-GPU configuration, at the top of the block-size range.

Metric: inverse roots per second of the whole job (all ranks), with the mean
step time beside it.  Timing: W untimed warm-up steps, then K steps, each
between two CUDA events on the launching stream, with a 256 MiB L2 flush
between steps outside the events; barrier + synchronize around the timed
region; max over ranks.  Multi-GPU runs shard the blocks of the one workload
across the ranks (strong scaling; shampoo_family_second_b200.sharded): every
rank holds its own local gradients, which are packed by block owner and
reduce-scattered over NCCL, steps the blocks it owns, and all-gathers the
updated blocks, so that every rank ends each step with the full weights.

The `e2e` figure repeats the timed steps through the public Python API with the
gradients in pinned host memory: each step copies them host -> device, runs
the step and reads the device status word back.  The copies run ahead of the
steps on a copy stream (a ring of device buffers), as a host-fed optimizer
prefetches its inputs.

`--impl reference` times the float64 CPU oracle (the only other program here)
on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np

import workloads

METRIC = "Shampoo step ms & inverse-roots/s at B=256..1024; % of tensor-core dense peak"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
TF32_PER_BF16 = 1.1 / 2.25   # nominal dense tf32 / bf16 tensor throughput ratio
SPLIT_PASSES = 3             # 3xTF32: three tf32 MMAs per fp32-accurate product
E2E_DEPTH = 4                # device input buffers the end-to-end pass prefetches into
WORKLOAD_NAMES = {
    "tiny": "tiny_64x32_b32",
    "lowrank": "lowrank_4x1024sq_b256",
    "gpt2": "gpt2_small_shapes_b512",
    "llama": "llama_1b_shapes_b1024",
    "sweep": "inverse_root_sweep",
    "soap": "soap_4x1024sq_b256",
    "tensor": "tensor_conv3x3_stack",
}
LLAMA_LAYER = 7  # weights per Llama layer (q, k, v, o, gate, up, down)


def workload_label(wl):
    """The workload's name; a Llama workload cut to fewer layers (--layers, for
    small profiling captures) says so."""
    name = WORKLOAD_NAMES.get(wl.name, wl.name)
    if wl.name == "llama" and len(wl.shapes) != len(workloads.WORKLOADS["llama"].shapes):
        name += f"_{len(wl.shapes) // LLAMA_LAYER}layers"
    return name


# Convolution kernels (3 x 3 x C_in x C_out) of a ResNet-style stack, for
# order-4 tensor Shampoo: 4 stages of 4 kernels at 64 .. 512 channels.
CONV_SHAPES = tuple((3, 3, c, c) for c in (64, 128, 256, 512) for _ in range(4))
SWEEP_BATCH = {256: 512, 512: 128, 1024: 64}
SOLVER_NAMES = {0: "coupled_newton", 1: "newton_db", 2: "chebyshev", 3: "coupled_newton_cubic",
                4: "coupled_newton_cubic_f64"}
SOLVER_IDS = {"newton": 0, "newton_db": 1, "chebyshev": 2, "newton_cubic": 3, "newton_cubic_f64": 4}
# fp64 tensor-core rate of a B200 (NVIDIA's nominal figure; no measured fp64 peak exists on this
# pool): the denominator of the fp64-iterate solver's product
FP64_NOMINAL_TFLOPS = 40.0


# ---------------------------------------------------------------------------
# shared helpers
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def max_over_ranks(values, world, device):
    """Elementwise maximum of per-rank timings; every rank must call it."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


BURST_WINDOW_MS = 1000.0     # a timed window shorter than this is compared with the burst peak


def tensor_peaks(peaks, window_ms):
    """fp32-equivalent 3xTF32 peaks (burst, sustained) from the bf16 figures,
    and which one a timed window of `window_ms` is compared with: the burst
    figure for a short window (the clocks have no time to settle under the
    power cap), the sustained one for a seconds-long window."""
    scale = TF32_PER_BF16 / SPLIT_PASSES
    burst = peaks["bf16_tflops"] * scale
    sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * scale
    return burst, sust, ("burst" if window_ms < BURST_WINDOW_MS else "sustained")


def job_throughput(units_per_rank, world, ms):
    """Whole-job rate of weak-scaled replicas: every rank processed
    `units_per_rank` units, the slowest in `ms` milliseconds."""
    return units_per_rank * world / (ms * 1e-3) if ms > 0 else 0.0


def refresh_steps(k, every):
    """Refresh steps in a window of k steps that starts on a refresh step."""
    return -(-k // every)


def phase_to_refresh(step, every):
    """First step >= `step` on which the roots are refreshed."""
    return -(-step // every) * every


def split_step_ms(step_ms, every):
    """Mean step time of the refresh steps and of the other steps of a window
    that starts on a refresh step (step k refreshes when k % every == 0)."""
    ref = [t for k, t in enumerate(step_ms) if k % every == 0]
    other = [t for k, t in enumerate(step_ms) if k % every != 0]
    return {"refresh_ms": sum(ref) / len(ref) if ref else None, "refresh_steps": len(ref),
            "non_refresh_ms": sum(other) / len(other) if other else None, "non_refresh_steps": len(other)}


class ClockSampler:
    """SM clocks and throttle reasons during the timed region.

    Polls NVML every ~2 ms from a thread (the timed regions are short); falls
    back to `nvidia-smi -lms 200` when NVML is unavailable."""

    REASONS = {  # NVML clocks-event reason bits
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4,
        "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.reason_bits = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self.thread = None
        self.proc = None
        self.lines = []

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = self.gpu
            if vis:
                ids = [v for v in vis.split(",") if v.strip()]
                if idx < len(ids) and ids[idx].strip().isdigit():
                    idx = int(ids[idx])
            h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)

            def poll():
                while not self._stop.is_set():
                    try:
                        self.samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
                        self.reason_bits |= pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    except Exception:
                        pass
                    time.sleep(0.002)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            return
        except Exception:
            pass
        try:
            fields = "clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown," \
                     "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap"
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={fields}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=lambda: self.lines.extend(l.strip() for l in self.proc.stdout),
                                           daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def stop(self):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for ln in self.lines:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 6:
                    continue
                try:
                    self.samples.append(float(parts[0]))
                    self.max_mhz = float(parts[1])
                except ValueError:
                    continue
                for nm, v in zip(names, parts[2:6]):
                    if v.lower() == "active":
                        self.reason_bits |= self.REASONS[nm]
        if self.thread is not None:
            self.thread.join(timeout=2)
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["no samples"], "samples": 0}
        reasons = sorted(k for k, bit in self.REASONS.items() if self.reason_bits & bit)
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def device_gradients(wl, seed, count, device):
    """`count` per-step gradient sets on the device, drawn with torch from the
    workload's recipe (same distribution as workloads.GradientStream)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    sets = []
    fixed = {}
    for i, (m, n) in enumerate(wl.shapes):
        if wl.name == "lowrank":
            fixed[i] = (torch.randn(m, 16, generator=g, device=device), torch.randn(n, 16, generator=g, device=device))
        elif wl.name == "gpt2":
            fixed[i] = 10.0 ** (torch.rand(n, generator=g, device=device) * 2.0 - 2.0)
    for _ in range(count):
        out = []
        for i, (m, n) in enumerate(wl.shapes):
            if wl.name == "lowrank":
                u, v = fixed[i]
                s = torch.randn(16, 16, generator=g, device=device)
                x = (u @ s @ v.T) / 16.0 + 0.01 * torch.randn(m, n, generator=g, device=device)
            elif wl.name == "gpt2":
                x = torch.randn(m, n, generator=g, device=device) * 0.02 * fixed[i][None, :]
            elif wl.name == "llama":
                x = (torch.randn(m, n, generator=g, device=device) * 0.01).to(torch.bfloat16)
            else:
                x = torch.randn(m, n, generator=g, device=device)
                if wl.grad_dtype == workloads.DTYPE_BF16:
                    x = x.to(torch.bfloat16)
            out.append(x.contiguous())
        sets.append(out)
    return sets


class ShardedRun:
    """The block-sharded step behind the interface the timing loop uses
    (step, status, step counter, block count of the whole job)."""

    def __init__(self, sb, wl, cfg, device):
        from shampoo_family_second_b200.sharded import ShardedShampoo
        self.inner = ShardedShampoo(wl.shapes, cfg, grads_reduced=False, device=device)
        self.local = self.inner.local_optimizer
        self.nb = len(self.inner.blocks)
        self.state = self.local.state if self.local is not None else None

    def step(self, W, G):
        self.inner.step(W, G)

    def status(self, reset=False):
        return self.local.status(reset) if self.local is not None else 0

    @property
    def step_count(self):
        return self.local.step_count if self.local is not None else 0

    def set_step_count(self, k):
        if self.local is not None:
            self.local.set_step_count(k)


def make_optimizer(sb, wl, cfg, world, device):
    """One GPU: the blocked step over every block.  Several: the blocks of the
    same workload sharded across the ranks."""
    if world == 1:
        return sb.Shampoo(wl.shapes, cfg, device=device)
    return ShardedRun(sb, wl, cfg, device)


def run_ours(args, wl):
    import torch
    import torch.distributed as dist
    import shampoo_family_second_b200 as sb

    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    cfg = sb.config_from_workload(wl)
    opt = make_optimizer(sb, wl, cfg, world, device)
    W = [torch.zeros(s, dtype=torch.float32, device=device) for s in wl.shapes]
    ring = max(1, min(args.ring, args.steps + args.warmup))
    grads = device_gradients(wl, wl.seed + 1000 * rank, ring, device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    nb = opt.nb
    roots_per_refresh = 2 * nb          # of the whole job (sharded runs split them across ranks)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    # warm-up
    for t in range(args.warmup):
        opt.step(W, grads[t % ring])
    barrier()
    if opt.status(reset=True) & ~(sb.DEVFLAG_NOT_CONVERGED | sb.DEVFLAG_STAGNATED):
        raise RuntimeError("device status reported an error during warm-up")

    # ---- timed region: K steps, per-step events, L2 flushed between steps
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    first = args.warmup
    opt.set_step_count(phase_to_refresh(first, wl.refresh_every))   # timed window starts on a refresh step
    launches0 = sb.launch_count()
    barrier()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        opt.step(W, grads[(first + k) % ring])
        ev[k][1].record(stream)
    barrier()
    launches = sb.launch_count() - launches0
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = float(sum(step_ms))
    nref = refresh_steps(args.steps, wl.refresh_every)
    status = opt.status(reset=True)

    # ---- roofline pass: same steps with per-launch events inside the library
    sb.profile_reset()
    sb.profile_enable(True)
    opt.set_step_count(phase_to_refresh(opt.step_count, wl.refresh_every))
    barrier()
    for k in range(args.steps):
        flush.zero_()
        opt.step(W, grads[(first + args.steps + k) % ring])
    barrier()
    tallies = {kind: sb.profile_read(kind) for kind in range(sb.KERNEL_KINDS)}
    sb.profile_enable(False)
    nref_prof = refresh_steps(args.steps, wl.refresh_every)

    # ---- end to end through the public API with host-resident gradients.
    # Every step copies its gradients from pinned host memory and reads the
    # device status word back.  Copies run ahead on a copy stream into a ring
    # of E2E_DEPTH device buffers (a step reuses a buffer only after the step
    # that consumed it), as an optimizer fed from the host prefetches its
    # inputs; before each copy the copy stream writes the 256 MiB flush buffer,
    # evicting L2 while earlier steps still run.
    depth = E2E_DEPTH
    set_bytes = sum(g.numel() * g.element_size() for g in grads[0])
    host = [[g.cpu().pin_memory() for g in gs] for gs in grads[: min(ring, 4 if set_bytes < (1 << 30) else 2)]]
    dev_in = [[torch.empty_like(g) for g in grads[0]] for _ in range(depth)]
    copy_stream = torch.cuda.Stream(device=device)
    copied = [torch.cuda.Event() for _ in range(depth)]
    consumed = [torch.cuda.Event() for _ in range(depth)]
    status_host = torch.zeros(max(args.steps, 1), dtype=torch.int32).pin_memory()
    h2d = sum(g.numel() * g.element_size() for g in host[0])
    status_view = (opt.state[:4].view(torch.int32) if opt.state is not None
                   else torch.zeros(1, dtype=torch.int32, device=device))
    opt.set_step_count(phase_to_refresh(opt.step_count, wl.refresh_every))
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)
    for k in range(args.steps):
        buf = k % depth
        with torch.cuda.stream(copy_stream):
            if k >= depth:
                copy_stream.wait_event(consumed[buf])
            flush.zero_()
            for d, h in zip(dev_in[buf], host[k % len(host)]):
                d.copy_(h, non_blocking=True)
            copied[buf].record(copy_stream)
        stream.wait_event(copied[buf])
        opt.step(W, dev_in[buf])
        status_host[k].copy_(status_view[0], non_blocking=True)
        consumed[buf].record(stream)
    e1.record(stream)
    e1.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    barrier()
    nref_e2e = refresh_steps(args.steps, wl.refresh_every)

    # ---- max over ranks
    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world, device)

    peaks, peak_src = load_peaks()
    g = tallies[sb.KERNEL_GEMM]
    gemm_avg_ms = g.total_ms / max(g.launches, 1)
    achieved = (g.alg_flops / max(g.launches, 1)) / (gemm_avg_ms * 1e-3) / 1e12 if g.launches else 0.0
    peak_burst, peak_sust, peak_kind = tensor_peaks(peaks, total_ms)
    peak = peak_burst if peak_kind == "burst" else peak_sust
    traffic = gemm_traffic_per_launch(wl)
    step_total_prof = sum(tl.total_ms for tl in tallies.values())
    roofline = {
        "kernel": "gemm3x_tf32_kernel",
        "bound": "tensor",
        "achieved": achieved,
        "peak": peak,
        "unit": "TFLOP/s",
        "frac": achieved / peak if peak else None,
        "traffic": traffic,
        "peak_kind": peak_kind,
        "frac_burst": achieved / peak_burst if peak_burst else None,
        "frac_sustained": achieved / peak_sust if peak_sust else None,
        "peak_basis": (f"{peak_src} bf16 {peak_kind} ({peaks['bf16_tflops']} burst, "
                       f"{peaks['bf16_tflops_sustained']} sustained TF/s) x {TF32_PER_BF16:.4f} "
                       f"(nominal tf32/bf16) / {SPLIT_PASSES} (3xTF32 passes): fp32-equivalent "
                       "algorithmic flops; frac is also the issued tf32 fraction; burst peak for a timed "
                       f"window under {BURST_WINDOW_MS:.0f} ms, sustained above"),
        "launches": g.launches, "avg_launch_ms": gemm_avg_ms,
        "share_of_step_kernel_time": g.total_ms / step_total_prof if step_total_prof else None,
        "refresh_steps": nref_prof,
    }
    d64 = tallies[sb.KERNEL_GEMM_F64]
    if d64.total_ms > g.total_ms:
        # fp64 statistics and iterates: the fp64 product dominates the step
        ach64 = d64.alg_flops / (d64.total_ms * 1e-3) / 1e12 if d64.total_ms > 0 else 0.0
        roofline = {
            "kernel": "dgemm_kernel", "bound": "tensor", "achieved": ach64, "peak": FP64_NOMINAL_TFLOPS,
            "unit": "TFLOP/s", "frac": ach64 / FP64_NOMINAL_TFLOPS, "traffic": None,
            "peak_basis": "nominal B200 fp64 tensor-core rate (not measured on this pool); executed fp64 flops",
            "launches": d64.launches, "avg_launch_ms": d64.total_ms / max(d64.launches, 1),
            "share_of_step_kernel_time": d64.total_ms / step_total_prof if step_total_prof else None,
            "refresh_steps": nref_prof,
            "gemm3x_tf32": {"achieved_tflops": achieved, "frac": achieved / peak if peak else None,
                            "peak_kind": peak_kind,
                            "share_of_step_kernel_time": g.total_ms / step_total_prof if step_total_prof else None},
        }

    fp64_mode = wl.solver == SOLVER_IDS["newton_cubic_f64"]
    rate = (lambda units, ms: units / (ms * 1e-3) if ms > 0 else 0.0)
    result = {
        "metric": METRIC,
        "value": rate(roots_per_refresh * nref, total_ms),
        "unit": "inverse-roots/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": total_ms / args.steps,
        "higher_is_better": True,
        "scaling": "strong",
        "vs_baseline": None,
        "dtype": "f64" if fp64_mode else "f32",
        "data": "synthetic",
        "config": {
            "workload": workload_label(wl),
            "params": len(wl.shapes), "param_elems": wl.n_params, "block": wl.block, "blocks": nb,
            "roots_per_refresh": roots_per_refresh, "refresh_every": wl.refresh_every,
            "refresh_steps_timed": nref, "solver": SOLVER_NAMES[wl.solver], "root_p": wl.root_p,
            "iters_cap": wl.iters, "tol": wl.tol, "beta": wl.beta, "eps": wl.eps, "momentum": wl.momentum,
            "grad_dtype": "bf16" if wl.grad_dtype == workloads.DTYPE_BF16 else "f32",
            "arithmetic": ("fp64 statistics and iterates (mma.sync f64), fp32 roots, 3xTF32 tcgen05 apply"
                           if fp64_mode else "3xTF32 tcgen05 (fp32-accurate), fp32 state"),
            "l2": "256 MiB buffer written between timed steps, outside the per-step events",
            "parallelism": (f"blocks sharded over {world} ranks (reduce-scatter of local gradients by block "
                            "owner, all-gather of updated blocks; NCCL)") if world > 1 else "single GPU",
        },
        "device_status": int(status),
        "gpu_launches": int(launches),
        "clocks": clk,
        "roofline": roofline,
        "kernels": {sb.KERNEL_NAMES[k]: {"launches": v.launches, "ms": round(v.total_ms, 4),
                                         "alg_tflop": round(v.alg_flops / 1e12, 6),
                                         "alg_gb": round(v.alg_bytes / 1e9, 6)}
                    for k, v in tallies.items() if v.launches},
        "e2e": {
            "value": rate(roots_per_refresh * nref_e2e, e2e_ms),
            "unit": "inverse-roots/s",
            "ms_per_step": e2e_ms / args.steps,
            "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": 4,
            "overlap": f"host-to-device copies (each after an L2 flush) run up to {E2E_DEPTH} steps ahead on a copy stream",
        },
    }
    result["step_ms_split"] = split_step_ms(step_ms, wl.refresh_every)   # this rank's timed steps
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, args.cpu_budget_s)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result), flush=True)


TRAFFIC_SOURCES = ("gemm_tc.cu", "solver.cu", "api.cu")


def code_only(text):
    """C++ source without comments and blank space (the traffic record tracks
    code, not its comments)."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    lines = []
    for line in text.splitlines():
        line = re.sub(r"//.*$", "", line).strip()
        if line:
            lines.append(" ".join(line.split()))
    return "\n".join(lines)


def traffic_source_sha(read=None):
    """sha256 over the code (comments dropped) of the sources that decide the
    GEMM launch mix of a step.  `read(name)` returns a source's text (default:
    the working tree)."""
    import hashlib
    if read is None:
        def read(name):
            with open(os.path.join(ROOT, "shampoo_family_second_b200", "csrc", name)) as f:
                return f.read()
    h = hashlib.sha256()
    for name in TRAFFIC_SOURCES:
        h.update(code_only(read(name)).encode())
    return h.hexdigest()


def gemm_traffic_per_launch(wl):
    """DRAM bytes per GEMM launch from the committed ncu capture of this
    workload's GEMMs, if the capture was taken on the current sources with the
    same workload and solver (else None)."""
    path = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if (d.get("source_sha256") != traffic_source_sha() or d.get("workload_key") != workload_label(wl)
                or d.get("solver") != SOLVER_NAMES[wl.solver]):
            return None
        return d.get("bytes_per_launch")
    except Exception:
        return None


# ---------------------------------------------------------------------------
# CPU baseline / reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------

def oracle_sample_plan(wl, budget_s):
    """Blocks and steps of a bounded oracle sample of the workload."""
    import oracle
    table = oracle.block_table(wl.shapes, wl.block)
    nb = len(table)
    # rough cost model of one eigh(B) + products, to keep the sample in budget
    per_block = 2 * (wl.block / 512.0) ** 3 * 0.06 + 1e-3
    n_blocks = max(1, min(nb, int(budget_s / max(per_block, 1e-4) / 2)))
    rng = np.random.default_rng(wl.seed)
    blocks = sorted(rng.choice(nb, size=n_blocks, replace=False).tolist())
    return blocks, nb


def time_oracle(wl, blocks, steps, warmup=0):
    import oracle
    params = sorted({oracle.block_table(wl.shapes, wl.block)[b].param for b in blocks})
    stream = workloads.GradientStream(wl, params=params)
    gen = []
    for _ in range(steps):
        gs = stream.next()
        full = [None] * len(wl.shapes)
        for p, g in zip(params, gs):
            full[p] = g
        gen.append(full)
    o = oracle.ShampooOracle(wl.shapes, wl.block, wl.beta, wl.eps, wl.lr, wl.root_p, wl.refresh_every,
                             blocks=blocks)
    times, nref = [], 0
    for t in range(steps):
        if t == warmup:
            o.t = phase_to_refresh(o.t, wl.refresh_every)   # timed window starts on a refresh step
        refresh = (o.t % wl.refresh_every) == 0
        t0 = time.perf_counter()
        o.step(gen[t])
        times.append(time.perf_counter() - t0)
        nref += int(refresh and t >= warmup)
    return times, nref


SINGLE_THREAD_WORKLOADS = ("tiny", "lowrank")


def single_thread_oracle(wl, blocks, nb, steps, est_s_per_block, budget_s):
    """The oracle over the same step window on one host thread (BLAS/LAPACK
    limited to one thread), on a prefix of the block sample sized so that even
    a run `cores` times slower than the multi-threaded one stays near
    budget_s; None when the thread limit cannot be set."""
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:
        return None
    k = max(1, min(len(blocks), int(budget_s / max(est_s_per_block, 1e-6))))
    sub = blocks[:k]
    with threadpool_limits(limits=1):
        times, nref = time_oracle(wl, sub, steps)
    return {"value": 2 * len(sub) * nref / sum(times), "unit": "inverse-roots/s", "cores": 1,
            "sample": (f"{len(sub)} of {nb} blocks, {steps} consecutive steps from step 0 ({nref} refresh), "
                       f"float64 numpy/LAPACK eigh, 1 thread")}


def cpu_baseline(wl, budget_s):
    cores = len(os.sched_getaffinity(0))
    blocks, nb = oracle_sample_plan(wl, budget_s)
    steps = min(wl.refresh_every, 10)
    times, nref = time_oracle(wl, blocks, steps)
    roots = 2 * len(blocks) * nref
    value = roots / sum(times)
    out = {"value": value, "unit": "inverse-roots/s", "cores": cores, "kind": "oracle",
           "sample": (f"{len(blocks)} of {nb} blocks, {steps} consecutive steps from step 0 "
                      f"({nref} refresh), float64 numpy/LAPACK eigh, {cores} host threads")}
    if wl.name in SINGLE_THREAD_WORKLOADS:
        per_block = sum(times) / len(blocks) * cores   # pessimistic one-thread time per block
        one = single_thread_oracle(wl, blocks, nb, steps, per_block, min(budget_s, 20.0) / 2.0)
        if one is not None:
            out["single_thread"] = one
    return out


def run_reference(args, wl):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    cores = len(os.sched_getaffinity(0))
    per_step_budget = max(1.0, args.cpu_budget_s / max(args.steps + args.warmup, 1))
    blocks, nb = oracle_sample_plan(wl, per_step_budget * wl.refresh_every)
    total = args.warmup + args.steps
    times, nref = time_oracle(wl, blocks, total, warmup=args.warmup)
    timed = times[args.warmup:]
    roots = 2 * len(blocks) * nref
    value = roots / sum(timed) if sum(timed) > 0 else 0.0
    sample = (f"{len(blocks)} of {nb} blocks per step, {args.steps} timed steps after {args.warmup} warm-up, "
              f"window starting on a refresh step ({nref} refresh), float64 numpy/LAPACK, {cores} host threads")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "inverse-roots/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(timed) / args.steps,
        "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES.get(wl.name, wl.name), "block": wl.block,
                   "refresh_every": wl.refresh_every, "sampled_blocks": len(blocks), "blocks": nb},
        "cpu_baseline": {"value": value, "unit": "inverse-roots/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "inverse-roots/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_other(args):
    """SOAP or order-4 tensor Shampoo through their C-ABI handles: W untimed
    and K timed steps, per-step CUDA events, the L2 flushed between steps.
    SOAP runs on the 4 x 1024^2 low-rank workload (block 256, refresh every
    10); tensor Shampoo on a stack of 3 x 3 convolution kernels (refresh every
    10).  Units: eigenbases (SOAP) or inverse roots (tensor) per second, with
    ms per step beside them."""
    import torch
    import shampoo_family_second_b200 as sb
    rank, world, _ = dist_env()
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    gen = torch.Generator(device=device)
    gen.manual_seed(77 + rank)
    if args.workload == "soap":
        wl = workloads.workload("lowrank")
        cfg = sb.make_config(wl.block, wl.beta, 0.0, 3e-3, refresh_every=wl.refresh_every)
        opt = sb.Soap(wl.shapes, cfg, sb.make_soap_config(jacobi_sweeps=15, refine_iters=1))
        shapes, every = wl.shapes, wl.refresh_every
        per_refresh = 2 * opt.nb
        grads = device_gradients(wl, wl.seed + 1000 * rank, min(args.ring, args.steps + args.warmup), device)
        unit = "eigenbases/s"
    else:
        shapes, every = CONV_SHAPES, 10
        cfg = sb.make_config(32, 0.999, 1e-6, 1e-3, solver=sb.SOLVER_NEWTON_CUBIC, iters=40, tol=1e-5,
                             refresh_every=every)
        opt = sb.TensorShampoo(shapes, cfg)
        per_refresh = sum(len(s) for s in shapes)
        grads = [[torch.randn(s, generator=gen, device=device) * 0.01 for s in shapes]
                 for _ in range(min(args.ring, args.steps + args.warmup))]
        unit = "inverse-roots/s"
    W = [torch.zeros(s, dtype=torch.float32, device=device) for s in shapes]
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for t in range(args.warmup):
        opt.step(W, grads[t % len(grads)])
    # the timed window starts on a refresh step
    k0 = args.warmup
    pad = (-k0) % every
    for t in range(pad):
        opt.step(W, grads[(k0 + t) % len(grads)])
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    l0 = sb.launch_count()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        opt.step(W, grads[(k0 + pad + k) % len(grads)])
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    launches = sb.launch_count() - l0
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total = sum(step_ms)
    nref = refresh_steps(args.steps, every)
    sb.profile_reset()
    sb.profile_enable(True)
    for k in range(args.steps):
        flush.zero_()
        opt.step(W, grads[k % len(grads)])
    torch.cuda.synchronize()
    tallies = {k: sb.profile_read(k) for k in range(sb.KERNEL_KINDS)}
    sb.profile_enable(False)
    g = tallies[sb.KERNEL_GEMM]
    peaks, src = load_peaks()
    pb, ps_, kind = tensor_peaks(peaks, total)
    ach = (g.alg_flops / g.launches) / (g.total_ms / g.launches * 1e-3) / 1e12 if g.launches else 0.0
    # the dominant kernel of these paths need not be the GEMM (the tensor step's permutes and
    # Gram sums, SOAP's Jacobi sweeps): report the roofline of whichever took the most time
    dom = max(tallies, key=lambda k: tallies[k].total_ms)
    if dom == sb.KERNEL_GEMM:
        peak = pb if kind == "burst" else ps_
        roofline = {"kernel": "gemm3x_tf32_kernel", "bound": "tensor", "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": ach / peak, "traffic": None,
                    "frac_burst": ach / pb, "frac_sustained": ach / ps_, "peak_kind": kind,
                    "launches": g.launches, "avg_launch_ms": g.total_ms / max(g.launches, 1),
                    "peak_basis": f"{src} bf16 {kind} x 1.1/2.25 / 3"}
    else:
        d = tallies[dom]
        gbs = d.alg_bytes / (d.total_ms * 1e-3) / 1e9 if d.total_ms > 0 else 0.0
        roofline = {"kernel": sb.KERNEL_NAMES[dom], "bound": "hbm", "achieved": gbs,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                    "launches": d.launches, "avg_launch_ms": d.total_ms / max(d.launches, 1),
                    "peak_basis": f"{src} copy bandwidth; algorithmic bytes of the kernel kind",
                    "gemm": {"achieved_tflops": ach, "frac_burst": ach / pb, "frac_sustained": ach / ps_}}
    kernels = {sb.KERNEL_NAMES[k]: {"launches": v.launches, "ms": round(v.total_ms, 4),
                                    "alg_tflop": round(v.alg_flops / 1e12, 6), "alg_gb": round(v.alg_bytes / 1e9, 6)}
               for k, v in tallies.items() if v.launches}
    status = opt.status()
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": per_refresh * nref / (total * 1e-3), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAMES[args.workload], "params": len(shapes),
                       "param_elems": int(sum(np.prod(s) for s in shapes)), "refresh_every": every,
                       "per_refresh": per_refresh, "refresh_steps_timed": nref,
                       "l2": "256 MiB buffer written between timed steps, outside the per-step events"},
            "step_ms_split": split_step_ms(step_ms, every), "device_status": int(status),
            "gpu_launches": int(launches), "clocks": clk, "roofline": roofline, "kernels": kernels,
        }), flush=True)


def run_sweep(args):
    """Inverse-root solver sweep: stacked fp32 SPD matrices Q diag(lam) Q^T
    (Haar Q, log-uniform lam with condition number kappa), one
    inv_root_batched call per step through the C ABI.  With --sweep-grid every
    (n, kappa, p, solver) of the sweep runs in turn, one JSON line each:
    n in {256, 512, 1024}, kappa in {1e2, 1e4, 1e6, 1e8}, p in {2, 4}; coupled
    Newton (both correction degrees) and Newton-DB residual-checked
    (tol 1e-5, cap 40), Chebyshev at degrees 16 and 32, and the fp64-iterate
    solver (tol 1e-12, cap 40)."""
    import torch
    import shampoo_family_second_b200 as sb

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group(backend="nccl", timeout=timedelta(seconds=120))
    device = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()
    if not args.sweep_grid:
        sweep_case(args, sb, device, stream, rank, world, args.sweep_n, args.sweep_kappa, args.sweep_p,
                   args.sweep_solver, args.sweep_iters, args.sweep_tol, args.sweep_degree)
    else:
        for n in (256, 512, 1024):
            for kappa in (1e2, 1e4, 1e6, 1e8):
                for p in (2, 4):
                    for name, degree in (("newton", 0), ("newton_cubic", 0), ("newton_db", 0),
                                         ("chebyshev", 16), ("chebyshev", 32), ("newton_cubic_f64", 0)):
                        tol = 0.0 if name == "chebyshev" else (1e-12 if name.endswith("f64") else 1e-5)
                        sweep_case(args, sb, device, stream, rank, world, n, kappa, p, name, 40, tol,
                                   degree or args.sweep_degree)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


_SWEEP_INPUT = {}


def sweep_case(args, sb, device, stream, rank, world, n, kappa, p, solver_name, sweep_iters, sweep_tol,
               sweep_degree):
    """One (n, kappa, p, solver) case of the sweep: W untimed and K timed calls."""
    import torch
    batch = args.sweep_batch or SWEEP_BATCH.get(n, 64)
    solver = SOLVER_IDS[solver_name]
    key = (batch, n, kappa, rank)
    if _SWEEP_INPUT.get("key") != key:  # the grid reuses one input set across p and solvers
        _SWEEP_INPUT.clear()
        _SWEEP_INPUT["key"] = key
        _SWEEP_INPUT["parts"] = workloads.spd_batch(batch, n, kappa, seed=4321 + n + rank, return_parts=True)
    A64, Q64, lam64 = _SWEEP_INPUT["parts"]
    A = torch.from_numpy(A64.astype(np.float32)).to(device)
    X = torch.empty_like(A)
    scratch = torch.empty(sb.inv_root_scratch_bytes(batch, n, solver), dtype=torch.uint8, device=device)
    iters = torch.zeros(batch, dtype=torch.int32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    lo = 0.999 / kappa if solver == 2 else 0.0
    kw = dict(p=p, eps=0.0, solver=solver, iters=sweep_iters, tol=sweep_tol, cheb_degree=sweep_degree,
              cheb_lo=lo, out=X, scratch=scratch, stream=stream)

    def one():
        _, it, st = sb.inv_root_batched(A, **kw)
        iters.copy_(it)
        status.copy_(st)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(device.index or 0)
    clocks.start()
    l0 = sb.launch_count()
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        one()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    launches = sb.launch_count() - l0
    clk = clocks.stop()
    total_ms = max_over_ranks([sum(a.elapsed_time(b) for a, b in ev)], world, device)[0]
    sb.profile_reset()
    sb.profile_enable(True)
    for k in range(args.steps):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    f64 = solver == SOLVER_IDS["newton_cubic_f64"]
    g = sb.profile_read(sb.KERNEL_GEMM_F64 if f64 else sb.KERNEL_GEMM)
    sb.profile_enable(False)
    peaks, src = load_peaks()
    peak_burst, peak_sust, peak_kind = tensor_peaks(peaks, total_ms)
    peak = peak_burst if peak_kind == "burst" else peak_sust
    ach = (g.alg_flops / g.launches) / (g.total_ms / g.launches * 1e-3) / 1e12 if g.launches else 0.0
    if f64:
        roofline = {"kernel": "dgemm_kernel", "bound": "tensor", "achieved": ach, "peak": FP64_NOMINAL_TFLOPS,
                    "unit": "TFLOP/s", "frac": ach / FP64_NOMINAL_TFLOPS, "traffic": None,
                    "launches": g.launches, "avg_launch_ms": g.total_ms / max(g.launches, 1),
                    "peak_basis": "nominal B200 fp64 tensor-core rate (not measured on this pool)"}
    else:
        roofline = {"kernel": "gemm3x_tf32_kernel", "bound": "tensor", "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": ach / peak if peak else None, "traffic": None,
                    "launches": g.launches, "avg_launch_ms": g.total_ms / max(g.launches, 1),
                    "peak_kind": peak_kind, "frac_burst": ach / peak_burst if peak_burst else None,
                    "frac_sustained": ach / peak_sust if peak_sust else None,
                    "peak_basis": f"{src} bf16 {peak_kind} x 1.1/2.25 / 3"}
    it_host = iters.cpu().numpy()
    # error of a few roots against the construction's own root Q lam^{-1/p} Q^T
    # (of the float64 matrix: includes the fp32 rounding of A, amplified ~kappa u / p)
    Xh = X.cpu().numpy().astype(np.float64)
    errs = []
    for i in range(min(2, batch)):
        ref = (Q64[i] * lam64[i] ** (-1.0 / p)) @ Q64[i].T
        errs.append(float(np.linalg.norm(Xh[i] - ref) / np.linalg.norm(ref)))
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": job_throughput(batch * args.steps, world, total_ms), "unit": "inverse-roots/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"inverse_root_sweep_{batch}x{n}sq_kappa{kappa:.0e}_p{p}_{solver_name}{sweep_degree if solver == 2 else ''}",
                       "n": n, "batch": batch, "kappa": kappa, "p": p, "solver": solver_name,
                       "iters": sweep_iters, "tol": sweep_tol, "degree": sweep_degree,
                       "l2": "256 MiB buffer written between timed calls, outside the events"},
            "iters_used": [int(it_host.min()), int(it_host.max())], "device_status": int(status.item()),
            "rel_err_vs_construction_sample": errs, "gpu_launches": int(launches), "clocks": clk,
            "roofline": roofline,
        }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama", choices=sorted(WORKLOAD_NAMES))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ring", type=int, default=8, help="distinct gradient sets kept on the device")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--solver", default=None, choices=sorted(SOLVER_IDS),
                    help="inverse-root solver of the step workloads (default: the workload's own)")
    ap.add_argument("--momentum", type=float, default=None, help="momentum ahead of the preconditioner (step workloads)")
    ap.add_argument("--layers", type=int, default=0,
                    help="Llama workload cut to its first N layers (small profiling captures; 0: all 16)")
    ap.add_argument("--sweep-n", type=int, default=512)
    ap.add_argument("--sweep-batch", type=int, default=0)
    ap.add_argument("--sweep-kappa", type=float, default=1e4)
    ap.add_argument("--sweep-p", type=int, default=4)
    ap.add_argument("--sweep-solver", default="newton", choices=sorted(SOLVER_IDS))
    ap.add_argument("--sweep-iters", type=int, default=25)
    ap.add_argument("--sweep-tol", type=float, default=0.0)
    ap.add_argument("--sweep-degree", type=int, default=32)
    ap.add_argument("--sweep-grid", action="store_true", help="run every (n, kappa, p, solver) case of the sweep")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload in ("soap", "tensor"):
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the SOAP and tensor workloads are timed for the "
                              "CUDA path only; the oracle arm covers the step workloads"}))
            return
        run_other(args)
        return
    if args.workload == "sweep":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the sweep is timed for the CUDA path only; "
                              "the oracle arm covers the step workloads"}))
            return
        run_sweep(args)
        return
    over = {}
    if args.solver is not None:
        over["solver"] = SOLVER_IDS[args.solver]
    if args.momentum is not None:
        over["momentum"] = args.momentum
    if args.layers:
        if args.workload != "llama":
            ap.error("--layers applies to the llama workload")
        over["shapes"] = workloads.WORKLOADS["llama"].shapes[:LLAMA_LAYER * args.layers]
    wl = workloads.workload(args.workload, **over)
    np.random.seed(0)
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
