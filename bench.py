"""Throughput benchmark: record + 10 gradient passes of a Lorenz ensemble.

One step = the whole hot path over one batch: gs_record (sizing pass, slot
ordering, recording pass) followed by 10 fused replay + reverse-sweep passes
(gs_grad) against the fixed mesh -- the workload "Lorenz (d=3), n = 2**20,
t in [0, 10], Tsit5 rtol = atol = 1e-6, ten save points with N(0,1) targets,
one record then ten gradient passes".  The metric is trajectory-gradients/s
over the whole step (record included).

  python bench.py [--gpus N --steps K --warmup W --dtype f64|f32 --impl ours|reference]

N > 1 runs under torchrun, one process per GPU; every rank owns its own
2**20 trajectories (weak scaling, no data-path collective: trajectories are
independent), timings are the max over ranks.  Inputs (mesh ~5 GB,
checkpoints ~14 GB per rank) are far larger than L2, so no flush is needed.
The CPU oracle appears twice: as ``cpu_baseline`` (a bounded sample timed on
the host cores, rank 0, N = 1) and as the whole ``--impl reference`` arm.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

PASSES = 10
# algorithmic flops of one Lorenz Tsit5 step: the forward replay step
# (12 add + 30 mul + 75 fma = 192) plus its transposed step (264, see DESIGN)
FLOP_FWD, FLOP_REV = 192, 264
FLOP_LOSS_PER_SAVE = 18  # 3 sub + 3 fma forward, 3 sub + 3 fma reverse
# FP64 peak derived from unit counts and clocks: 148 SMs x 64 FP64 FMA/clk x 2
FP64_PEAK = 148 * 64 * 2 * 1965e6
FP32_PEAK = 148 * 128 * 2 * 1965e6


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--dtype", default="f64", choices=["f64", "f32"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--n", type=int, default=None, help="trajectories per GPU (default 2**20)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_{os.getpid()}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "200"]
            if bus_id:
                cmd += ["-i", bus_id]
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
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
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)), "reasons": sorted(reasons),
                "samples": len(sm)}


def bus_id_of(dev) -> str | None:
    import torch
    try:
        pr = torch.cuda.get_device_properties(dev)
        return f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
    except Exception:
        return None


def cpu_baseline(prob_full, sample: int):
    """The oracle as it stands: record + one gradient pass of a sample, on the
    host cores; scaled to the step's 1 record + 10 passes."""
    import oracle
    sub = prob_full.subset(np.arange(sample))
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    om = oracle.record(sub, 2048, nthreads=threads)
    t1 = time.perf_counter()
    oracle.grad(sub, om, nthreads=threads)
    t2 = time.perf_counter()
    per_step = (t1 - t0) + PASSES * (t2 - t1)
    return {"value": sample * PASSES / per_step, "unit": "trajectory-gradients/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{sample} of the {prob_full.n} trajectories: oracle record {t1 - t0:.2f} s + one tape "
                      f"gradient pass {t2 - t1:.2f} s, scaled to 1 record + {PASSES} passes"}


def run_reference(args):
    """--impl reference: the CPU oracle on the host cores, same metric/config."""
    import oracle
    import workloads
    rank, world, _ = dist_env()
    if rank != 0:
        return
    n_full = args.n or (1 << 20)
    sample = 256
    prob = workloads.lorenz_1m(sample, dtype=args.dtype)
    threads = oracle.default_threads()
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        om = oracle.record(prob, 2048, nthreads=threads)
        for _ in range(PASSES):
            oracle.grad(prob, om, nthreads=threads)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    t = float(np.mean(times))
    value = sample * PASSES / t
    line = {"impl": "reference", "metric": "trajectory-gradients/s (Lorenz fp64, 1M traj)", "value": value,
            "unit": "trajectory-gradients/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": args.dtype, "data": "synthetic",
            "config": {"workload": f"lorenz_1m: Lorenz d=3, n={n_full} per GPU, t in [0,10], Tsit5 rtol=atol=1e-6, "
                                   f"10 save points, 1 record + {PASSES} gradient passes",
                       "sample_per_step": sample},
            "cpu_baseline": {"value": value, "unit": "trajectory-gradients/s", "cores": threads, "kind": "oracle",
                             "sample": f"{sample} trajectories per step (record + {PASSES} tape gradient passes)"},
            "e2e": {"value": value, "unit": "trajectory-gradients/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    import workloads
    import discrete_adjoint_b200 as gs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    n = args.n or (1 << 20)
    prob = workloads.lorenz_1m(n, dtype=args.dtype, seed_offset=rank)
    td = torch.float64 if args.dtype == "f64" else torch.float32
    esz = 8 if args.dtype == "f64" else 4
    stream = torch.cuda.current_stream()

    # host inputs (pinned) and their device copies
    h_p = torch.from_numpy(np.ascontiguousarray(prob.p)).to(td).pin_memory()
    h_u0 = torch.from_numpy(np.ascontiguousarray(prob.u0)).to(td).pin_memory()
    h_tg = torch.from_numpy(np.ascontiguousarray(prob.target)).to(td).pin_memory()
    d_p, d_u0, d_tg = h_p.to(dev), h_u0.to(dev), h_tg.to(dev)
    ens = gs.Ensemble("lorenz", "tsit5", args.dtype, d_p, d_u0, prob.t0, prob.t1, [float(x) for x in prob.tsave])

    # sizing pass (setup, untimed): mesh capacity = the longest chain
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 4096)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(n, smax, len(prob.tsave), args.dtype, dev)
    ws_rec = gs.workspace(gs.gs_workspace_bytes(ens, mesh, gs.gradsolve.OP_RECORD), dev)
    ws_grad = gs.workspace(gs.gs_workspace_bytes(ens, mesh, gs.gradsolve.OP_GRAD), dev)
    outs = [gs.new_grad_out(ens) for _ in range(2)]

    ev = lambda: torch.cuda.Event(enable_timing=True)
    grad_events = []
    rec_events = []

    def step(timing):
        e0 = ev() if timing else None
        if timing:
            e0.record(stream)
        gs.gs_record(ens, mesh, prob.rtol, prob.atol, ws=ws_rec, stream=stream)
        if timing:
            e1 = ev()
            e1.record(stream)
            rec_events.append((e0, e1))
        for k in range(PASSES):
            if timing:
                a = ev()
                a.record(stream)
            gs.gs_grad(ens, mesh, "sumsq", target=d_tg, out=outs[k % 2], ws=ws_grad, stream=stream)
            if timing:
                b = ev()
                b.record(stream)
                grad_events.append((a, b))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step(False)
    barrier()
    clk = ClockSampler(bus_id_of(dev))
    launches0 = gs.gs_launch_count()
    barrier()
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
    t_end.record(stream)
    barrier()
    launches = gs.gs_launch_count() - launches0
    clocks = clk.stop()
    elapsed = t_start.elapsed_time(t_end) / 1e3
    grad_ms = float(np.mean([a.elapsed_time(b) for a, b in grad_events]))
    rec_ms = float(np.mean([a.elapsed_time(b) for a, b in rec_events]))
    tmax = torch.tensor([elapsed, grad_ms, rec_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
    elapsed, grad_ms, rec_ms = tmax.tolist()

    # end to end through the public API from host buffers: H2D of the inputs,
    # the record, and per pass the gradient plus a D2H read of (loss, dp, du0)
    h_loss = torch.empty(n, dtype=td).pin_memory()
    h_dp = torch.empty((3, n), dtype=td).pin_memory()
    h_du0 = torch.empty((3, n), dtype=td).pin_memory()

    def e2e_step():
        d_p.copy_(h_p, non_blocking=True)
        d_u0.copy_(h_u0, non_blocking=True)
        d_tg.copy_(h_tg, non_blocking=True)
        gs.gs_record(ens, mesh, prob.rtol, prob.atol, ws=ws_rec, stream=stream)
        for k in range(PASSES):
            o = outs[k % 2]
            gs.gs_grad(ens, mesh, "sumsq", target=d_tg, out=o, ws=ws_grad, stream=stream)
            h_loss.copy_(o.loss, non_blocking=True)
            h_dp.copy_(o.dp, non_blocking=True)
            h_du0.copy_(o.du0, non_blocking=True)

    e2e_steps = max(1, min(args.steps, 3))
    e2e_step()
    barrier()
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    barrier()
    e2e_t = torch.tensor([a.elapsed_time(b) / 1e3 / e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    h2d = (h_p.numel() + h_u0.numel() + h_tg.numel()) * esz
    d2h = PASSES * (h_loss.numel() + h_dp.numel() + h_du0.numel()) * esz

    # algorithmic work of one gradient launch
    total_steps = int(mesh.nsteps.sum().item())
    flops = (FLOP_FWD + FLOP_REV) * total_steps + FLOP_LOSS_PER_SAVE * len(prob.tsave) * n
    achieved = flops / (grad_ms / 1e3)
    peak = FP64_PEAK if args.dtype == "f64" else FP32_PEAK
    ns = mesh.nsteps.double()
    value = world * n * PASSES * args.steps / elapsed
    line = {
        "metric": "trajectory-gradients/s (Lorenz fp64, 1M traj)" if args.dtype == "f64"
        else "trajectory-gradients/s (Lorenz fp32, 1M traj)",
        "value": value, "unit": "trajectory-gradients/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": {"workload": f"lorenz_1m: Lorenz d=3, n={n} per GPU, t in [0,10], Tsit5 rtol=atol=1e-6, "
                               f"10 save points with N(0,1) targets, 1 record + {PASSES} gradient passes per step",
                   "n_per_gpu": n, "passes_per_step": PASSES, "smax": smax,
                   "steps_total": total_steps, "steps_mean": float(ns.mean()),
                   "steps_max_over_mean": float(ns.max() / ns.mean()),
                   "grad_ms": grad_ms, "record_ms": rec_ms,
                   "grad_only_value": world * n / (grad_ms / 1e3),
                   "l2": "inputs larger than L2 (mesh %.1f GB, checkpoints %.1f GB); no flush" % (
                       mesh.h.numel() * esz / 1e9, ws_grad.numel() / 1e9),
                   "parallelism": f"dp{world} (independent trajectory shards)"},
        "clocks": clocks,
        "e2e": {"value": world * n * PASSES / float(e2e_t.item()), "unit": "trajectory-gradients/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "roofline": {"bound": "alu", "achieved": achieved / 1e12, "peak": peak / 1e12, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "kernel": "k_grad_tsit5_lorenz", "peak_source": "derived: 148 SMs x %d FMA/clk x 2 x 1965 MHz"
                     % (64 if args.dtype == "f64" else 128),
                     "flops_per_launch": flops},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(prob, 2048)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
