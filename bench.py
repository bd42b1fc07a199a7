#!/usr/bin/env python
"""Benchmark of libgspn's 4-direction GSPN forward on one B200 per process.

Default workload: N=16, C=8, H=W=1024, all four directions summed, channel-shared weights
(logits N x 1 x 3 x H x W per direction) with per-channel lambda and u, fp32 storage.

A step is one full forward (all directions, weight formation, injection, merge and gate)
over one batch of synthetic input already resident in HBM. ``value`` is the compulsory HBM
throughput of the whole job: (x, lambda, u read once + logits read once + y written once) x
number of ranks / max-over-ranks device time. The inputs (2.95 GB per rank) are larger than L2,
so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libgspn|reference]

Under torchrun (N > 1) every rank runs its own batch (weak scaling, no collective on the data
path); timing is bracketed by a barrier and a device synchronise and the max over ranks is
reported. ``--impl reference`` times the float64 CPU oracle instead, on bounded samples of the
same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gspn_inputs  # noqa: E402

METRIC = "4-dir GSPN scan fwd ms & achieved HBM GB/s (frac of peak), 1024² B16 C8"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic_highres.md")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="libgspn", choices=["libgspn", "reference"])
    ap.add_argument("--workload", default="highres", choices=sorted(gspn_inputs.WORKLOADS) + ["all"],
                    help="'all': one line per workload, in the order tiny, classifier, highres, wide, train")
    ap.add_argument("--shard", action="store_true",
                    help="strong scaling: split the workload's planes over the ranks (batch blocks, else channel "
                         "blocks) instead of giving every rank the whole workload")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-planes", type=int, default=24, help="planes of the CPU oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="also time the backward (gradients of x, logits, lambda, u); on by default for 'train'")
    ap.add_argument("--proxy", type=int, default=0,
                    help="compressive channel proxy: project C channels to this many, propagate, project back")
    ap.add_argument("--chunk", type=int, default=0,
                    help="local propagation: lines per chunk along each scan axis (0 = global, the metric's)")
    ap.add_argument("--algo", default="auto", choices=["auto", "generic", "plane", "sweep", "band"],
                    help="kernel family (auto: the library's choice)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch N (small cases for profiler captures; not a bench line)")
    ap.add_argument("--height", type=int, default=0,
                    help="override the workload's map height H (small cases for profiler captures; not a bench line)")
    return ap.parse_args()


def env_rank():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def dtype_name(wl):
    return "f32" if wl.dtype == "f32" else "bf16"


def config_of(wl, world, chunk=0):
    return {
        "workload": wl.name,
        "N": wl.N, "C": wl.C, "H": wl.H, "W": wl.W,
        "directions": "TB+BT+LR+RL" if wl.mask == 15 else wl.mask,
        "weights": "channel-shared" if wl.wmode else "per-channel",
        "storage": wl.dtype,
        "per_rank_batch": wl.N,
        "global_batch": wl.N * world,
        "parallelism": f"dp{world}" if world > 1 else "single",
        "l2": ("inputs larger than L2 (no flush)" if wl.compulsory_fwd_bytes() > 126 * 2 ** 20
               else "inputs fit in L2: a parity-size case, not a bandwidth figure"),
        "chunk": chunk,
    }


# --------------------------------------------------------------------------- CPU oracle sample
def oracle_plane_seconds_only(wl, planes, chunk=0):
    """Oracle time excluding input generation."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(1)
    H, W, D = wl.H, wl.W, wl.D
    x = rng.standard_normal((1, 1, H, W))
    a = rng.standard_normal((D, 1, 1, 3, H, W)) * wl.a_std
    lam = rng.uniform(0, 1, (1, 1, H, W))
    u = rng.standard_normal((1, 1, H, W))
    t0 = time.perf_counter()
    for _ in range(planes):
        oracle.forward(x, a, lam, u, wl.wmode, wl.mask, chunk=chunk)
    return time.perf_counter() - t0


def plane_bytes(wl):
    return (4 * wl.H * wl.W + (wl.D * 3 * wl.H * wl.W) // (wl.C if wl.wmode else 1)) * wl.elem_bytes


def host_cpu():
    """(logical cores, CPU model) of this host."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count(), model


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return
    names = ["tiny", "classifier", "highres", "wide", "train"] if args.workload == "all" else [args.workload]
    for name in names:
        reference_line(args, gspn_inputs.WORKLOADS[name], world)


def reference_line(args, wl, world):
    planes_per_step = 2
    times = []
    for s in range(args.warmup + args.steps):
        dt = oracle_plane_seconds_only(wl, planes_per_step, args.chunk)
        if s >= args.warmup:
            times.append(dt)
    tot = sum(times)
    nbytes = plane_bytes(wl) * planes_per_step * len(times)
    value = nbytes / tot / 1e9
    ms_per_step = tot / len(times) * 1e3
    nproc, model = host_cpu()
    line = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "ms_per_full_forward_extrapolated": round(ms_per_step * (wl.N * wl.C) / planes_per_step, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": config_of(wl, world, args.chunk),
        "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": 1, "host_nproc": nproc,
                         "cpu_model": model, "kind": "oracle",
                         "sample": f"{planes_per_step} of {wl.N * wl.C} (n,c) planes per step (ms_per_step is "
                                   "the measured time of that sample), float64 C oracle, one thread"},
        "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- clocks sampler
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"gspn_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in open(self.path):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# Sources of the kernels the traffic summary describes (the sweep family and its device
# helpers); host-side entry points and the other families do not change their traffic.
SWEEP_SOURCES = ("gspn_common.cuh", "sweep_io.cuh", "k_sweep.cu")


def kernel_source_sha():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_spatial_propagation_gspn_b200", "csrc")
    for fn in SWEEP_SOURCES:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload):
    """DRAM traffic per forward from the committed ncu summary (its 'traffic-json:' line), if the
    kernel sources are unchanged since the capture: (bytes per forward, bytes per launch)."""
    if workload != "highres" or not os.path.exists(TRAFFIC_FILE):
        return None, None
    d = None
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if line.startswith("traffic-json:"):
                d = json.loads(line[len("traffic-json:"):])
    if not d or d.get("source_sha") != kernel_source_sha():
        return None, None
    return d.get("dram_bytes_per_forward"), d.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- GPU arm
def run_libgspn(args):
    import torch
    import torch.distributed as dist

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    names = ["tiny", "classifier", "highres", "wide", "train"] if args.workload == "all" else [args.workload]
    for name in names:
        line = bench_workload(args, name, rank, local_rank, world)
        if rank == 0:
            print(json.dumps(line), flush=True)
        torch.cuda.empty_cache()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def _max_over_ranks(v, world, dev):
    import torch
    import torch.distributed as dist
    if world == 1:
        return v
    tt = torch.tensor([v], device=dev, dtype=torch.float64)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def bench_workload(args, name, rank, local_rank, world):
    import torch
    import torch.distributed as dist
    import linear_spatial_propagation_gspn_b200 as g
    from linear_spatial_propagation_gspn_b200 import sharding

    wl = gspn_inputs.WORKLOADS[name]
    if args.batch:
        wl = wl.with_(N=args.batch)
    if args.height:
        wl = wl.with_(H=args.height)
    dev = torch.device("cuda", local_rank)
    full_wl = wl
    shard = None
    if args.shard:
        # strong scaling: every rank draws the same full inputs and keeps its plane shard
        t = gspn_inputs.make_inputs(wl, device=dev)
        shard = sharding.plan(wl.N, wl.C, world, rank)
        shared = wl.wmode == 1
        t = {k: (sharding.take(v, shard, logits=(k == "a"), shared=shared).contiguous()) for k, v in t.items()}
        wl = wl.with_(N=t["x"].shape[0], C=t["x"].shape[1])
        torch.cuda.empty_cache()
    else:
        t = gspn_inputs.make_inputs(wl, device=dev, seed=wl.seed + 1000 * rank)
    x, a, lam, u = t["x"], t["a"], t["lam"], t["u"]
    algo_req = {"auto": g.ALGO_AUTO, "generic": g.ALGO_GENERIC, "plane": g.ALGO_PLANE, "sweep": g.ALGO_SWEEP,
                "band": g.ALGO_BAND}[args.algo]
    desc = g.desc_for(x, wl.wmode, wl.mask, algo=algo_req, chunk=args.chunk)
    algo = g.selected_algo(desc)
    ws = g.alloc_workspace(desc, False, dev)
    y = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    def step():
        g.forward(x, a, lam, u, wl.wmode, wl.mask, algo=algo_req, y=y, ws=ws, chunk=args.chunk)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if g.device_status(ws) != g.GSPN_OK:
        raise RuntimeError("device status reports a timeout during warm-up")

    # ---- timed region: K steps, one event per step boundary on the launching stream
    sampler = ClockSampler(local_rank)
    sampler.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    evs[0].record(stream)
    for k in range(args.steps):
        step()
        evs[k + 1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms_total = _max_over_ranks(evs[0].elapsed_time(evs[-1]), world, dev)
    per_step = [evs[k].elapsed_time(evs[k + 1]) for k in range(args.steps)]
    ms_median = _max_over_ranks(statistics.median(per_step), world, dev)
    ms_step = ms_total / args.steps
    comp = wl.compulsory_fwd_bytes()
    job_bytes = full_wl.compulsory_fwd_bytes() if args.shard else comp * world
    job_elems = full_wl.numel if args.shard else wl.numel * world
    value = job_bytes / (ms_step * 1e-3) / 1e9

    # ---- per-kernel timing pass (events recorded by the library around each launch)
    nk = 8
    kevs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * nk)]
    for e in kevs:
        e.record(stream)  # materialise the event handles
    torch.cuda.synchronize()
    reps = max(5, min(50, args.steps // 4))
    per = None
    launches = 0
    for _ in range(reps):
        launches = g.forward_timed(x, a, lam, u, y, ws, desc, kevs)
        torch.cuda.synchronize()
        d = [kevs[2 * k].elapsed_time(kevs[2 * k + 1]) for k in range(launches)]
        per = d if per is None else [p + q for p, q in zip(per, d)]
    per = [p / reps for p in per]
    peak, peak_kind = measured_peak()
    kern_ms = sum(per)
    names = launch_names(wl, algo, launches)
    achieved = comp / (kern_ms * 1e-3) / 1e9
    traffic, per_launch = (committed_traffic(wl.name) if not (args.batch or args.height or args.shard)
                           else (None, None))
    roofline = {
        "bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
        "frac": round(achieved / peak, 4), "traffic": traffic,
        "peak_kind": peak_kind,
        "what": (f"whole forward = {launches} launches ({'+'.join(names)}); algorithmic bytes = compulsory "
                 f"x, lam, u, a read once + y written once = {comp} B per forward; time = sum of the launches"),
        "kernels_ms": {n: round(p, 4) for n, p in zip(names, per)} if len(names) == len(per) else [round(p, 4) for p in per],
    }
    if per_launch and len(per_launch) == len(per):
        # DRAM bytes each launch moves (ncu) over its event-timed duration
        roofline["kernels_dram_gbs"] = {n: round(b / (p * 1e-3) / 1e9, 1) for n, b, p in zip(names, per_launch, per)}

    # ---- backward (A7): gradients of sum(dy * y), timed on its own
    bwd = None
    if args.backward or wl.name == "train":
        dy = torch.randn(x.shape, generator=torch.Generator(device=dev).manual_seed(wl.seed + 7), device=dev,
                         dtype=torch.float32).to(x.dtype)
        bdesc = g.desc_for(x, wl.wmode, wl.mask, chunk=args.chunk)
        bws = g.alloc_workspace(bdesc, True, dev)
        outs = (torch.empty_like(x), torch.empty_like(a), torch.empty_like(x), torch.empty_like(x))

        def bstep():
            g.backward(x, a, lam, u, dy, wl.wmode, wl.mask, out=outs, ws=bws, chunk=args.chunk)

        for _ in range(max(3, args.warmup // 2)):
            bstep()
        torch.cuda.synchronize()
        nb_steps = max(5, args.steps // 4)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        bev = [torch.cuda.Event(enable_timing=True) for _ in range(nb_steps + 1)]
        bev[0].record(stream)
        for k in range(nb_steps):
            bstep()
            bev[k + 1].record(stream)
        torch.cuda.synchronize()
        bms = _max_over_ranks(bev[0].elapsed_time(bev[-1]) / nb_steps, world, dev)
        bmed = _max_over_ranks(statistics.median(bev[k].elapsed_time(bev[k + 1]) for k in range(nb_steps)),
                               world, dev)
        bcomp = wl.compulsory_bwd_bytes()
        bjob = full_wl.compulsory_bwd_bytes() if args.shard else bcomp * world
        bgbs = bjob / (bms * 1e-3) / 1e9
        bwd = {"ms_per_step": round(bms, 4), "ms_median": round(bmed, 4), "steps": nb_steps,
               "compulsory_bytes": bcomp, "value": round(bgbs, 2), "unit": "GB/s",
               "frac": round(bcomp / (bms * 1e-3) / 1e9 / peak, 4),
               "algo": g.ALGO_NAMES.get(g.selected_algo(bdesc, True), "?"),
               "what": "reads dy, x, lambda, u, logits; writes dx, dlambda, du, dlogits (compulsory bytes)",
               "train_step_ms": round(ms_step + bms, 4)}
        # the training pair: a forward that keeps each direction's h and a backward that reads it
        # instead of recomputing the scans (where the library runs it), timed as whole steps
        hsz = g.hsave_size(bdesc) if not args.chunk else 0
        if hsz > 0:
            hsave = torch.empty(hsz // 4, dtype=torch.float32, device=dev)
            ysv = torch.empty_like(x)

            def pstep():
                g.forward_save(x, a, lam, u, wl.wmode, wl.mask, y=ysv, hsave=hsave, ws=ws)
                g.backward_saved(x, a, lam, u, dy, hsave, wl.wmode, wl.mask, out=outs, ws=bws)

            for _ in range(max(3, args.warmup // 2)):
                pstep()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            pev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            pev[0].record(stream)
            for _ in range(nb_steps):
                pstep()
            pev[1].record(stream)
            torch.cuda.synchronize()
            pms = _max_over_ranks(pev[0].elapsed_time(pev[1]) / nb_steps, world, dev)
            bwd["train_step_saved_h_ms"] = round(pms, 4)
            bwd["train_step_saved_h_what"] = ("forward that keeps each direction's h + backward that reads it "
                                              "(gspn_forward_save, gspn_backward_saved), per step")
            del hsave, ysv
        del bws, outs, dy

    # ---- copy ceiling on the same byte volume
    nb = (comp // 2) // 16 * 16
    src = torch.empty(nb, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    for _ in range(3):
        g.copy_ceiling(src, dst)
    c0 = torch.cuda.Event(enable_timing=True)
    c1 = torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(10):
        g.copy_ceiling(src, dst)
    c1.record(stream)
    torch.cuda.synchronize()
    copy_gbs = 2 * nb * 10 / (c0.elapsed_time(c1) * 1e-3) / 1e9
    del src, dst

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        hx, ha, hl, hu = (tt.cpu().pin_memory() for tt in (x, a, lam, u))
        hy = torch.empty(x.shape, dtype=x.dtype).pin_memory()
        dev_buf = torch.empty(g.forward_host_buffer_size(desc), dtype=torch.uint8, device=dev)
        g.forward_host(desc, hx, ha, hl, hu, hy, dev_buf)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        q0 = torch.cuda.Event(enable_timing=True)
        q1 = torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        for _ in range(args.e2e_steps):
            g.forward_host(desc, hx, ha, hl, hu, hy, dev_buf)
        q1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = _max_over_ranks(q0.elapsed_time(q1) / args.e2e_steps, world, dev)
        h2d = sum(tt.numel() * tt.element_size() for tt in (hx, ha, hl, hu))
        d2h = hy.numel() * hy.element_size()
        e2e = {"value": round(job_bytes / (e2e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "api": "gspn_forward_host (pinned host buffers)"}
        del dev_buf, hx, ha, hl, hu, hy

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        planes = min(args.cpu_planes, wl.N * wl.C)
        secs = oracle_plane_seconds_only(wl, planes, args.chunk)
        nproc, model = host_cpu()
        cpu = {"value": round(plane_bytes(wl) * planes / secs / 1e9, 6), "unit": "GB/s", "cores": 1,
               "host_nproc": nproc, "cpu_model": model, "kind": "oracle",
               "output_elements_per_s": round(planes * wl.H * wl.W / secs, 1),
               "sample": f"{planes} of {wl.N * wl.C} (n,c) planes, float64 C oracle, one thread, "
                         f"{secs:.1f} s"}

    del t, x, a, lam, u, y, ws
    if world > 1:
        dist.barrier()
    return {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms_step, 4),
        "ms_median": round(ms_median, 4),
        "output_elements_per_s": round(job_elems / (ms_step * 1e-3), 1),
        "higher_is_better": True, "scaling": "strong" if args.shard else "weak", "vs_baseline": None,
        "dtype": dtype_name(wl), "data": "synthetic (seeded torch.randn/rand on device)",
        "config": dict(config_of(full_wl, 1 if args.shard else world, args.chunk),
                       **({"shard": f"{shard.axis}[{shard.start}:{shard.stop}] on rank 0",
                           "parallelism": f"{shard.axis.lower()}-shard{world}"} if args.shard else {})),
        "algo": g.ALGO_NAMES.get(algo, str(algo)),
        "roofline": roofline,
        "copy_ceiling_gbs": round(copy_gbs, 1),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "backward": bwd,
        "gpu_launches": launches * args.steps,
        "clocks": clocks,
    }


def launch_names(wl, algo, launches):
    if algo == 4:   # band family
        return ["weights", "TB-ckpt+z", "LR-ckpt", "BT+TB-recompute", "RL+LR-recompute"][:launches]
    dirs = [n for n, bit in zip(("TB", "BT", "LR", "RL"), (1, 2, 4, 8)) if wl.mask & bit]
    if launches == len(dirs) + 1:
        return ["weights"] + dirs
    if launches == 1:
        return ["plane" if algo == 2 else "forward"]
    return [f"launch{k}" for k in range(launches)]


def run_proxy(args):
    """Compressive channel proxy on the named workload: x has the workload's C channels, the
    propagation runs on args.proxy channels (logits, lambda and u in proxy space), the two
    projections are GEMMs on the tensor cores. Reports the whole proxied forward and, timed
    separately, its propagation alone."""
    import torch
    import linear_spatial_propagation_gspn_b200 as g
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = gspn_inputs.WORKLOADS[args.workload]
    if args.batch:
        wl = wl.with_(N=args.batch)
    if args.height:
        wl = wl.with_(H=args.height)
    Cp = args.proxy
    pw = wl.with_(C=Cp)
    t = gspn_inputs.make_inputs(wl, device=dev)
    tp = gspn_inputs.make_inputs(pw, device=dev, seed=wl.seed + 17)
    x = t["x"]
    a, lam, u = tp["a"], tp["lam"], tp["u"]
    gen = torch.Generator(device=dev).manual_seed(wl.seed + 29)
    p_in = (torch.randn(Cp, wl.C, generator=gen, device=dev) / wl.C ** 0.5).to(x.dtype)
    p_out = (torch.randn(wl.C, Cp, generator=gen, device=dev) / Cp ** 0.5).to(x.dtype)
    y = torch.empty_like(x)
    desc = g.make_desc(wl.N, Cp, wl.H, wl.W, wl.wmode, wl.mask, g._dtype_code(x.dtype), chunk=args.chunk)
    ws = torch.empty(int(g.lib().gspn_proxy_workspace_size(desc, wl.C)), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        g.proxy_forward(x, p_in, a, lam, u, p_out, wl.wmode, wl.mask, y=y, ws=ws, chunk=args.chunk)

    def timed(fn, k):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(k):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / k

    sampler = ClockSampler(0)
    sampler.start()
    time.sleep(0.3)
    ms = timed(step, args.steps)
    clocks = sampler.stop()
    xp = tp["x"]
    yp = torch.empty_like(xp)
    sws = g.alloc_workspace(g.desc_for(xp, wl.wmode, wl.mask, chunk=args.chunk), False, dev)
    scan_ms = timed(lambda: g.forward(xp, a, lam, u, wl.wmode, wl.mask, y=yp, ws=sws, chunk=args.chunk),
                    max(5, args.steps // 2))
    es = wl.elem_bytes
    hw = wl.H * wl.W
    comp = (2 * wl.N * wl.C * hw + 2 * wl.N * Cp * hw + 2 * Cp * wl.C + a.numel()) * es
    flops = 2 * 2 * wl.N * hw * wl.C * Cp
    peak, peak_kind = measured_peak()
    line = {
        "metric": METRIC, "variant": f"compressive channel proxy {wl.C} -> {Cp} channels",
        "value": round(comp / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_name(wl), "data": "synthetic (seeded torch.randn/rand on device)",
        "config": dict(config_of(wl, 1, args.chunk), proxy=Cp),
        "proxy": {"C": wl.C, "C_proxy": Cp, "scan_ms": round(scan_ms, 4),
                  "projections_ms": round(ms - scan_ms, 4), "projection_tflop_per_step": round(flops / 1e12, 4),
                  "projection_tflops": round(flops / ((ms - scan_ms) * 1e-3) / 1e12, 1) if ms > scan_ms else None,
                  "compulsory_bytes": comp,
                  "what": "x read and y written at C channels; lambda, u, logits at C_proxy; P_in, P_out"},
        "roofline": {"bound": "hbm", "achieved": round(comp / (ms * 1e-3) / 1e9, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(comp / (ms * 1e-3) / 1e9 / peak, 4), "traffic": None, "peak_kind": peak_kind},
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.proxy and args.workload == "all":
        raise SystemExit("--proxy runs one named workload")
    if args.impl == "reference":
        run_reference(args)
    elif args.proxy:
        run_proxy(args)
    else:
        run_libgspn(args)


if __name__ == "__main__":
    main()
