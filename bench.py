#!/usr/bin/env python
"""Throughput of the B200 Muon / Dimuon step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload large_batch|large_batch_dimuon|large_batch_quarter|gpt2_small|
                               square1024|square4096|lora_r2|lora_r8|lora_r32|
                               vec_w1|vec_w2|vec_w8|vec_w32|vec_w128]
                    [--no-cpu-baseline] [--debug-flags BITS] [--sharded]

Defaults: 50 timed steps after 10 warm-ups, the large batch, one GPU.

--sharded times the data-parallel form instead of replicas: ONE copy of the
workload split over the N ranks by whole matrices (dimuon_optimizer_b200.sharded:
balanced ownership, flat rank-contiguous buffers); each step is the
reduce-scatter of every rank's local gradients (NCCL), the library step on the
owned matrices and the all-gather of the updated weights (NCCL).  Strong
scaling: `value` is the workload's matrices per second; the line also gives
the exchange's own time.

One step = one optimizer step (momentum, normalisation, five Newton-Schulz
iterations, scale, decay, apply) over every matrix of the workload.  The
default workload is the large batch: 8 x 4096^2, 4 x 4096x14336 and
4 x 14336x4096 bf16 matrices (tall ones orthogonalised on their short side),
Muon mode, bf16 tensor-core products with fp32 accumulation.

Each rank runs its own copy of the workload on its own GPU (independent
problems, no collective on the data path): weak scaling; `value` counts the
matrices of all ranks.  Rank 0 prints one JSON line.

Workloads whose buffers fit a few times in L2 (126 MB) are timed step by
step with a 512 MB buffer written between the steps (outside the timed
events), so every step starts with a cold L2; the large ones run back to
back (their inputs are larger than L2).
"""
import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "Muon/Dimuon step matrices/s and NS5 TFLOP/s on B200 (% of bf16 / HBM roofline)"


def workload_spec(name):
    if name == "large_batch":
        return dict(shapes=workloads.large_batch_shapes(), cond=False, mdt="bf16", lr=0.02,
                    wd=0.0, moonshot=False, seed=3,
                    desc="8x4096^2 + 4x4096x14336 + 4x14336x4096 bf16, Muon, 5 NS5 iterations")
    if name == "large_batch_dimuon":  # the large batch through the Dimuon path
        return dict(shapes=[(4096, 4096)] * 8 + [(4096, 14336)] * 4 + [(14336, 4096)] * 4,
                    cond=True, mdt="bf16", lr=0.02, wd=0.0, moonshot=False, seed=3,
                    desc="8x4096^2 + 4x4096x14336 + 4x14336x4096 bf16, Dimuon, 5 NS5 iterations")
    if name == "large_batch_quarter":  # same shapes, a quarter of the matrices
        return dict(shapes=[(4096, 4096)] * 2 + [(4096, 14336), (14336, 4096)], cond=False,
                    mdt="bf16", lr=0.02, wd=0.0, moonshot=False, seed=3,
                    desc="2x4096^2 + 4096x14336 + 14336x4096 bf16, Muon, 5 NS5 iterations")
    if name == "gpt2_small":
        return dict(shapes=workloads.gpt2_small_shapes(), cond=False, mdt="bf16", lr=0.02,
                    wd=0.1, moonshot=True, seed=2,
                    desc="GPT-2-small hidden matrices (72) bf16, Muon, Moonshot scale, wd 0.1")
    if name == "square1024":
        return dict(shapes=workloads.single_square_shapes(), cond=False, mdt="bf16", lr=0.02,
                    wd=0.0, moonshot=False, seed=1, desc="one 1024x1024 bf16 matrix, Muon")
    if name == "square4096":
        return dict(shapes=workloads.single_square_shapes(4096), cond=False, mdt="bf16",
                    lr=0.02, wd=0.0, moonshot=False, seed=1,
                    desc="one 4096x4096 bf16 matrix, Muon, 5 NS5 iterations")
    if name == "toy":  # the 4x16 toy factor; latency-bound, read as microseconds per step
        return dict(shapes=[(4, 16)], cond=True, mdt="fp32", lr=0.02, wd=0.0, moonshot=False,
                    seed=0, desc="one 4x16 factor (bf16 W/G, fp32 M), Dimuon; latency-bound")
    if name.startswith("lora_r"):
        r = int(name[6:])
        return dict(shapes=workloads.lora_shapes(r), cond=True, mdt="fp32",
                    lr={2: 0.018, 8: 0.010, 32: 0.010}.get(r, 0.01), wd=0.0, moonshot=False,
                    seed=4, desc=f"224 LoRA projections r={r} (A r x 4096, B 4096 x r), "
                                 "fp32 momentum, bf16 weights, Dimuon")
    if name.startswith("vec_w"):
        w = int(name[5:])
        return dict(shapes=workloads.vector_shapes(w), cond=False, mdt="fp32", lr=0.02, wd=0.0,
                    moonshot=False, seed=5, nesterov=1, vec_len=workloads.VECTOR_LENGTH,
                    desc=f"{workloads.VECTOR_COUNT} 1-D parameters of {workloads.VECTOR_LENGTH} "
                         f"variables at width {w} (zero-padded), fp32 momentum, bf16 weights, "
                         "Muon with Nesterov")
    raise SystemExit(f"unknown workload {name}")


def ns_flops(shapes):
    """Algorithmic Newton-Schulz flops per iteration: 3 m^2 n + m^3 per matrix
    (symmetric products counted once), m the short side."""
    tot = 0.0
    for r, c in shapes:
        m, n = min(r, c), max(r, c)
        tot += 3.0 * m * m * n + m ** 3
    return tot


def step_bytes(spec):
    """Algorithmic HBM bytes of one step outside the products: read G, read
    and write M, read and write W."""
    mb = 4 if spec["mdt"] == "fp32" else 2
    return sum(r * c for r, c in spec["shapes"]) * (2 + 2 * mb + 4)


def thin_fp64_flops(spec, thin_max=32, split_r32=False):
    """Algorithmic fp64 flops of the thin-factor path per step: per long-side
    column of a factor with short side r, the Gram sums S_1 (and S_2 when
    conditioned), r (r + 1) / 2 multiply-adds each, and O = T b, r^2; two
    flops per multiply-add.  (The r x r iteration is O(r^3) per factor.)
    With split_r32 (bf16 tensor-core mode) the r = 32 factors take those sums
    on bf16 tensor cores and add no fp64 work."""
    tot = 0.0
    for rows, cols in spec["shapes"]:
        r, n = min(rows, cols), max(rows, cols)
        if r > thin_max or (split_r32 and r == 32):
            continue
        tot += 2.0 * n * (r * (r + 1) / 2 * (2 if spec["cond"] else 1) + r * r)
    return tot


# fp64 fused multiply-adds per clock of one B200 SM (NVIDIA's 40 TF/s fp64 figure:
# 148 SMs x 64 FMA x 2 flops at the boost clock)
FP64_FMA_PER_SM_CLK = 64


# DRAM traffic of the tensor-core product per launch (ncu dram__bytes_read.sum +
# dram__bytes_write.sum of the quarter batch, same shapes, scaled by 4), averaged
# over the three products of a middle iteration (the launches the live timing
# isolates), valid only for the kernel build the ncu capture was taken from.
TRAFFIC_CAPTURED = {"large_batch": 2459e6}
TRAFFIC_BUILD = "e6b8acca114dcfd4"
TRAFFIC_SOURCES = ["k_ns_tc2.cu", "dm_tc_epilogue.cuh", "dm_sm100.cuh"]


def kernel_build_hash():
    import hashlib
    parts = []
    for f in TRAFFIC_SOURCES:
        with open(os.path.join(ROOT, "dimuon_optimizer_b200", "csrc", f), "rb") as fh:
            parts.append(hashlib.sha256(fh.read()).hexdigest())
    return hashlib.sha256("".join(parts).encode()).hexdigest()[:16]


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            return json.load(fh), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
         "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        return parse_clock_log(out)


def parse_clock_log(text):
    """Summary of nvidia-smi samples (the ClockSampler query, csv, no header,
    no units): median SM clock and the throttle reasons seen while the GPU
    was busy (utilisation >= 50 %; all samples if none was)."""
    rows = []
    for ln in text.strip().splitlines():
        f = [x.strip() for x in ln.split(",")]
        if len(f) < 10:
            continue
        try:
            rows.append(dict(sm=float(f[1]), smax=float(f[2]), util=float(f[4]),
                             hw=f[6], hwt=f[7], swt=f[8], pcap=f[9]))
        except ValueError:
            continue
    load = [r for r in rows if r["util"] >= 50] or rows
    if not load:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
    reasons = set()
    for r in load:
        for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                        ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
            if r[k].lower() == "active":
                reasons.add(name)
    return {"sm_mhz": float(np.median([r["sm"] for r in load])),
            "sm_max_mhz": max(r["smax"] for r in load), "reasons": sorted(reasons),
            "samples": len(load)}


L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 512 * 2 ** 20


def resident_bytes(spec):
    """Bytes of the buffers one step touches: G, M, W and the fp32 update
    each once (the workspace is extra)."""
    mb = 4 if spec["mdt"] == "fp32" else 2
    return sum(r * c for r, c in spec["shapes"]) * (2 + mb + 2)


def l2_flushed(spec):
    return resident_bytes(spec) < 3 * L2_BYTES


def config_of(spec, world, precision="bf16"):
    """The workload description both arms print."""
    cfg = {"workload": spec["desc"], "matrices": len(spec["shapes"]),
           "parallelism": f"replica per GPU x{world}",
           "l2": ("512 MB written between timed steps (per-step CUDA events)" if l2_flushed(spec)
                  else "inputs larger than L2 (no flush)")}
    if precision == "fp32":
        cfg["products"] = "fp32 (DM_PREC_FP32)"
    return cfg


def interleaved_order(shapes):
    """Matrix indices with the shape classes interleaved (a, b, c, a, b, c,
    ...), so that any run of consecutive steps samples every class."""
    classes = {}
    for i, s in enumerate(shapes):
        classes.setdefault(s, []).append(i)
    order, lists = [], list(classes.values())
    while any(lists):
        for lst in lists:
            if lst:
                order.append(lst.pop(0))
    return order


def oracle_run(spec, idx, ns_steps=5):
    """Seconds the fp64 CPU oracle takes for one step of matrix `idx` of the
    workload (input draws excluded)."""
    import oracle as orc
    shp = spec["shapes"][idx]
    rng = np.random.default_rng(spec["seed"] + idx)
    G = rng.standard_normal(shp)
    W = 0.02 * rng.standard_normal(shp)
    M = np.zeros(shp)
    h = orc.HParams(lr=spec["lr"], weight_decay=spec["wd"], ns_steps=ns_steps,
                    nesterov=bool(spec.get("nesterov", 0)),
                    scale_mode=orc.SCALE_MOONSHOT if spec["moonshot"] else orc.SCALE_NONE)
    t0 = time.perf_counter()
    if spec["cond"]:
        orc.dimuon_step(W, G, M, np.zeros(shp[0]), np.zeros(shp[1]), h,
                        momentum_dtype=spec["mdt"], weight_dtype="bf16")
    else:
        orc.muon_step(W, G, M, h, momentum_dtype=spec["mdt"], weight_dtype="bf16")
    return time.perf_counter() - t0


def cpu_baseline(spec):
    """The oracle's time for one whole step of the workload, measured per
    shape class: one matrix of each (short side, long side) class is run
    through the full 5-iteration step (a tall matrix is the transposed wide
    one for the oracle) and the step time is the sum over the workload's
    matrices of their class's time."""
    classes = {}
    for i, (r, c) in enumerate(spec["shapes"]):
        classes.setdefault((min(r, c), max(r, c)), []).append(i)
    total = 0.0
    for key, members in classes.items():
        total += len(members) * oracle_run(spec, members[0])
    names = ", ".join(f"{len(m)} x {k[0]}x{k[1]}" for k, m in classes.items())
    return total, (f"one matrix of each shape class ({names}) timed through the whole "
                   f"5-iteration step; the step time is the sum over all "
                   f"{len(spec['shapes'])} matrices of their class's time")


def reference_budget(spec):
    """Matrices per reference step: as many consecutive matrices (in the
    interleaved order) as make about 2e12 algorithmic flops, at least one."""
    per = 5 * ns_flops(spec["shapes"]) / len(spec["shapes"])
    return max(1, int(2e12 // max(per, 1.0)))


def run_reference(args, spec, rank, world):
    """The fp64 oracle as it stands, on the host cores, rank 0 only: each step
    runs the next few matrices of the workload (interleaved shape classes,
    cyclically) through the whole step; value = matrices processed / time."""
    if rank != 0:
        return
    threads = os.cpu_count()
    order = interleaved_order(spec["shapes"])
    per_step = min(reference_budget(spec), len(order))
    pos = 0

    def one_step():
        nonlocal pos
        dt = 0.0
        for _ in range(per_step):
            dt += oracle_run(spec, order[pos % len(order)])
            pos += 1
        return dt

    for _ in range(args.warmup):
        one_step()
    t = sum(one_step() for _ in range(args.steps))
    value = per_step * args.steps / t
    sample = (f"{per_step} matrix(es) of the workload per step, taken in turn with the shape "
              f"classes interleaved, each through the whole 5-iteration step (fp64 oracle)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "matrices/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(spec, world, args.precision),
            "cpu_baseline": {"value": value, "unit": "matrices/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "matrices/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def sharded_line(spec, world, steps, warmup, t_step, t_exchange, plan_loads, clocks, launches,
                 slice_elems=0):
    """JSON line of the --sharded mode (strong scaling over `world` ranks).
    Exchange bytes per rank and step: the reduce-scatter sends and the
    all-gather receives world - 1 bf16 slices each."""
    n_mat = len(spec["shapes"])
    cfg = config_of(spec, world)
    cfg["parallelism"] = (f"whole-matrix sharding over {world} rank(s): reduce-scatter of "
                          f"gradients, library step on owned matrices, all-gather of weights")
    return {"metric": METRIC, "value": n_mat / t_step, "unit": "matrices/s", "n_gpus": world,
            "steps": steps, "warmup": warmup, "ms_per_step": t_step * 1e3,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded N(0,1) gradients, N(0,0.02^2) weights)",
            "config": cfg, "exchange_ms_per_step": t_exchange * 1e3,
            "exchange_bytes_per_step": 2 * (world - 1) * slice_elems * 2,
            "plan_load_s": plan_loads, "clocks": clocks,
            "gpu_launches": launches, "mode": "sharded"}


def run_sharded(args, spec, rank, world, local):
    import datetime

    import torch
    import torch.distributed as dist

    import dimuon_optimizer_b200 as dm
    from dimuon_optimizer_b200 import sharded

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    shapes = spec["shapes"]
    plan = sharded.plan_shards(shapes, world)
    mdt = torch.float32 if spec["mdt"] == "fp32" else torch.bfloat16
    sw = sharded.ShardedWeights(plan, dtype=torch.bfloat16, device=dev)
    sg = sharded.ShardedGrads(plan, dtype=torch.bfloat16, device=dev)
    torch.manual_seed(spec["seed"] + 1000)
    sw.flat.copy_((0.02 * torch.randn(sw.flat.numel(), device=dev)).to(torch.bfloat16))
    own = plan.owned(rank)
    M = {i: torch.zeros(shapes[i], dtype=mdt, device=dev) for i in own}
    ER = {i: torch.zeros(shapes[i][0], device=dev) for i in own} if spec["cond"] else None
    EC = {i: torch.zeros(shapes[i][1], device=dev) for i in own} if spec["cond"] else None
    g_local = torch.Generator(device=dev)
    g_local.manual_seed(spec["seed"] + 17 * rank)
    local_grads = torch.randn(sg.flat.numel(), generator=g_local, device=dev).to(torch.bfloat16)
    hp = dm.dm_default_hparams(lr=spec["lr"], weight_decay=spec["wd"],
                               scale_mode=dm.DM_SCALE_MOONSHOT if spec["moonshot"]
                               else dm.DM_SCALE_NONE, nesterov=spec.get("nesterov", 0))
    nbytes = sharded.workspace_bytes(sw, rank, sg.views, M, hp, spec["cond"], ER, EC)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)

    owned = sharded.owned_matrices(sw, rank, sg, M, conditioned=spec["cond"], row_energy=ER,
                                   col_energy=EC)

    def step():
        sg.flat.copy_(local_grads)  # this rank's backward output
        sharded.sharded_step(sw, rank, sg, M, hp, ws, conditioned=spec["cond"], row_energy=ER,
                             col_energy=EC, mats=owned)

    def exchange_only():
        sg.reduce(rank)
        sw.gather(rank)

    def timed(fn, reps):
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        t = e0.elapsed_time(e1) / 1e3
        if world > 1:
            x = torch.tensor([t], dtype=torch.float64, device=dev)
            dist.all_reduce(x, op=dist.ReduceOp.MAX)
            t = float(x.item())
        return t

    for _ in range(args.warmup):
        step()
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    t_step = timed(step, args.steps) / args.steps
    clocks = sampler.stop()
    t_ex = timed(exchange_only, args.steps) / args.steps
    loads = [plan.load(q) for q in range(world)]
    launches = 0
    if own:
        launches = dm.dm_step_launches(
            [dm.dm_matrix(sw.views[i], sg.views[i], M[i], ER[i] if ER else None,
                          EC[i] if EC else None) for i in own], hp, int(spec["cond"]))
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(sharded_line(spec, world, args.steps, args.warmup, t_step, t_ex, loads,
                                      clocks, launches * args.steps, plan.slice_elems)),
              flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="large_batch")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--debug-flags", type=lambda v: int(v, 0), default=0,
                    help="library debug_flags (test hooks such as DM_DBG_TC_SINGLE; none skips "
                         "work)")
    ap.add_argument("--precision", default="bf16", choices=["bf16", "fp32"],
                    help="Newton-Schulz products on bf16 tensor cores (default) or fp32 SIMT")
    ap.add_argument("--sharded", action="store_true",
                    help="one workload sharded over the ranks (strong scaling) instead of replicas")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    spec = workload_spec(args.workload)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, spec, rank, world)
        return
    if args.sharded:
        run_sharded(args, spec, rank, world, local)
        return

    import torch
    import torch.distributed as dist

    import dimuon_optimizer_b200 as dm

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    shapes = spec["shapes"]
    bf = torch.bfloat16
    mdt = torch.float32 if spec["mdt"] == "fp32" else bf
    rng = np.random.default_rng(spec["seed"] + 17 * rank)
    torch.manual_seed(spec["seed"] + 1000 + rank)
    # gradients: views into one flat buffer on each side (each matrix starts on
    # a 128-byte boundary), so a step's host-to-device copy is a single copy
    offs, tot = [], 0
    for (r, c) in shapes:
        offs.append(tot)
        tot += (r * c + 63) // 64 * 64
    G_host_flat = torch.zeros(tot, dtype=bf).pin_memory()
    G_flat = torch.empty(tot, dtype=bf, device=dev)
    G, W, M, ER, EC = [], [], [], [], []
    for (r, c), o in zip(shapes, offs):
        gn = rng.standard_normal((r, c), dtype=np.float32)
        if spec.get("vec_len"):  # 1-D parameter: zero gradient in the padding cells
            gn.reshape(-1)[spec["vec_len"]:] = 0.0
        G_host_flat[o:o + r * c].view(r, c).copy_(torch.from_numpy(gn).to(bf))
        G.append(G_flat[o:o + r * c].view(r, c))
        W.append((0.02 * torch.randn((r, c), device=dev, dtype=torch.float32)).to(bf))
        M.append(torch.zeros((r, c), device=dev, dtype=mdt))
        ER.append(torch.zeros(r, device=dev, dtype=torch.float32) if spec["cond"] else None)
        EC.append(torch.zeros(c, device=dev, dtype=torch.float32) if spec["cond"] else None)
    G_flat.copy_(G_host_flat)
    mats = [dm.dm_matrix(W[i], G[i], M[i], ER[i], EC[i]) for i in range(len(shapes))]
    prec = dm.DM_PREC_FP32 if args.precision == "fp32" else dm.DM_PREC_BF16_TC
    hp = dm.dm_default_hparams(lr=spec["lr"], weight_decay=spec["wd"],
                               scale_mode=dm.DM_SCALE_MOONSHOT if spec["moonshot"]
                               else dm.DM_SCALE_NONE, nesterov=spec.get("nesterov", 0),
                               debug_flags=args.debug_flags, precision=prec)
    step_fn = dm.dm_dimuon_step if spec["cond"] else dm.dm_muon_step
    ws = torch.empty(dm.dm_workspace_size(mats, hp, int(spec["cond"])), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.Stream(device=dev)

    def capture(h):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            dm.check(step_fn(mats, h, ws, stream=stream))
        return g

    # warm-up eagerly once (plans, tensor maps), then capture the step
    with torch.cuda.stream(stream):
        dm.check(step_fn(mats, hp, ws, stream=stream))
    torch.cuda.synchronize(dev)
    graph = capture(hp)

    flush = l2_flushed(spec)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flush else None

    def timed(g, reps):
        """Device seconds of `reps` replays on the launch stream: one event
        pair around all of them, or (small workloads) one pair per replay with
        L2 flushed before each, outside the events."""
        barrier()
        torch.cuda.synchronize(dev)
        if not flush:
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                e0.record(stream)
                for _ in range(reps):
                    g.replay()
                e1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            return e0.elapsed_time(e1) / 1e3
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        with torch.cuda.stream(stream):
            for a, b in evs:
                flush_buf.fill_(1)
                a.record(stream)
                g.replay()
                b.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        return sum(a.elapsed_time(b) for a, b in evs) / 1e3

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize(dev)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    sampler.start()
    t_dev = max_over_ranks(timed(graph, args.steps))
    clocks = sampler.stop()
    ms_step = t_dev / args.steps * 1e3
    n_mat = len(shapes)
    value = world * n_mat * args.steps / t_dev

    # dominant kernel (tensor-core product): 4 extra iterations of a 5-step
    # schedule over a 1-step schedule, on the launch stream
    reps = max(2, min(args.steps, 5))
    hp1 = dm.dm_default_hparams(lr=spec["lr"], weight_decay=spec["wd"], ns_steps=1,
                                scale_mode=hp.scale_mode, nesterov=hp.nesterov,
                                debug_flags=args.debug_flags, precision=prec)
    g1 = capture(hp1)
    g1.replay()
    t5 = timed(graph, reps) / reps
    t1 = timed(g1, reps) / reps
    del g1
    per_iter_flops = ns_flops([s for s in shapes if min(s) > dm.DM_THIN_MAX])
    peaks, peak_kind = load_peaks()
    tc_launches = 3 * 4
    if per_iter_flops > 0 and t5 > t1 and args.precision == "fp32":
        # fp32 SIMT products: bound by the FMA pipes, 148 SMs x 128 fp32 lanes x 2
        # flops per clock at the sampled SM clock (74.5 TF/s at 1965 MHz)
        achieved = 4 * per_iter_flops / (t5 - t1) / 1e12
        mhz = clocks.get("sm_mhz") or 1965.0
        peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        roofline = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None, "kernel": "simt_ns_product",
                    "avg_launch_ms": (t5 - t1) / tc_launches * 1e3,
                    "peak_kind": f"derived fp32 FMA peak at the sampled {mhz:.0f} MHz"}
    elif per_iter_flops > 0 and t5 > t1:
        achieved = 4 * per_iter_flops / (t5 - t1) / 1e12
        # the sustained figure (a seconds-long loop under the power cap) when
        # the timed region ran power-capped, else the burst figure
        capped = "sw_power_cap" in (clocks.get("reasons") or [])
        peak = (peaks.get("bf16_tflops_sustained", 1400.0) if capped
                else peaks.get("bf16_tflops", 1590.0))
        traffic = None
        if args.workload in TRAFFIC_CAPTURED and kernel_build_hash() == TRAFFIC_BUILD:
            traffic = TRAFFIC_CAPTURED[args.workload]
        roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "kernel": "tc_ns_product_pair" if args.workload.startswith("large_batch")
                    else "tc_ns_product(_pair)",
                    "avg_launch_ms": (t5 - t1) / tc_launches * 1e3,
                    "peak_kind": f"{peak_kind} bf16 dense, "
                                 f"{'sustained (run power-capped)' if capped else 'burst'}"}
    else:
        gbs = step_bytes(spec) / (ms_step / 1e3) / 1e9
        peak = peaks.get("hbm_gbs", 6650.0)
        per_step = dm.dm_step_launches(mats, hp, int(spec["cond"]))
        label = ("thin_cluster (the whole step in one launch per 448 factors)"
                 if per_step <= -(-len(shapes) // 448) else
                 "thin path (thin_setup, thin_gram, thin_iterate, thin_apply; or thin_fused)")
        # the bound is the slower floor: the step's algorithmic bytes at the HBM
        # copy rate, or its fp64 arithmetic at the fp64 FMA rate (r = 32 in fp32
        # mode; in bf16 mode those sums run on bf16 tensor cores)
        mhz = clocks.get("sm_mhz") or 1965.0
        f64_peak = 148 * FP64_FMA_PER_SM_CLK * 2 * mhz * 1e6 / 1e12
        flops = thin_fp64_flops(spec, split_r32=args.precision == "bf16")
        if flops / (f64_peak * 1e12) > step_bytes(spec) / (peak * 1e9):
            roofline = {"bound": "alu", "achieved": flops / (ms_step / 1e3) / 1e12,
                        "peak": f64_peak, "unit": "TFLOP/s",
                        "frac": flops / (ms_step / 1e3) / 1e12 / f64_peak, "traffic": None,
                        "kernel": label + ": algorithmic fp64 flops of the whole step over the "
                                          "step time",
                        "launches_per_step": per_step, "hbm_GBps": gbs, "hbm_frac": gbs / peak,
                        "peak_kind": f"derived fp64 FMA peak at the sampled {mhz:.0f} MHz"}
        else:
            roofline = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s",
                        "frac": gbs / peak, "traffic": None,
                        "kernel": label + ": algorithmic bytes of the whole step over the step "
                                          "time",
                        "launches_per_step": per_step,
                        "peak_kind": f"{peak_kind} HBM copy"}

    # end to end through the public API: every step's gradients copied in from
    # pinned host memory, its status word read back.  Two device gradient sets:
    # step t + 1's host-to-device copy runs on its own stream while step t
    # computes; a step waits for its copy, and a copy waits until the step that
    # last read its buffer has finished.
    h2d = G_host_flat.numel() * G_host_flat.element_size()
    G2_flat = torch.empty_like(G_flat)
    G2 = [G2_flat[o:o + r * c].view(r, c) for (r, c), o in zip(shapes, offs)]
    bufs = [G_flat, G2_flat]
    mats_buf = [mats, [dm.dm_matrix(W[i], G2[i], M[i], ER[i], EC[i]) for i in range(len(shapes))]]
    cstream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]

    def h2d_copy(t):
        b = t % 2
        with torch.cuda.stream(cstream):
            if t >= 2:
                cstream.wait_event(consumed[b])
            bufs[b].copy_(G_host_flat, non_blocking=True)
            copied[b].record(cstream)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        cstream.wait_event(e0)
        h2d_copy(0)
        for t in range(args.steps):
            b = t % 2
            stream.wait_event(copied[b])
            dm.check(step_fn(mats_buf[b], hp, ws, stream=stream))
            consumed[b].record(stream)
            if t + 1 < args.steps:
                h2d_copy(t + 1)
            st = dm.dm_read_device_status(ws, stream=stream)
            assert st == dm.DM_OK, dm.dm_status_string(st)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3)
    e2e = {"value": world * n_mat * args.steps / t_e2e, "unit": "matrices/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 4,
           "h2d_overlap": "step t+1's copy overlaps step t (two device gradient sets)"}
    del G2, G2_flat, mats_buf
    del graph
    if world > 1:
        dist.destroy_process_group()

    if rank != 0:
        return
    launches = dm.dm_step_launches(mats, hp, int(spec["cond"]))
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        full, sample = cpu_baseline(spec)
        cpu = {"value": n_mat / full, "unit": "matrices/s", "cores": os.cpu_count(),
               "kind": "oracle", "sample": sample}
    line = {"metric": METRIC, "value": value, "unit": "matrices/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if args.precision == "fp32" else "bf16",
            "data": "synthetic (seeded N(0,1) gradients, N(0,0.02^2) weights)",
            "config": config_of(spec, world, args.precision), "cuda_graph": True,
            "ns_tflops_step": ns_flops(shapes) * hp.ns_steps / (ms_step / 1e3) / 1e12,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks,
            "gpu_launches": launches * args.steps}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
