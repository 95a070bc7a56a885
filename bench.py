"""Throughput benchmark of the record-and-replay gradient path.

One step = the whole hot path over one batch of synthetic input: a record of
the ensemble (one adaptive pass into the mesh) followed by the workload's
gradient passes (fused replay + reverse sweep, gs_grad) against the fixed
mesh.  Setup records the ensemble once with gs_record (adaptive pass, slot
sort by step count, gather into slot order); each step then re-records it in
that slot order with gs_record_inplace, straight into the mesh (--record full:
gs_record in every step).  The default workload is "Lorenz (d=3), n = 2**20 per GPU, t in
[0, 10], Tsit5 rtol = atol = 1e-6, ten save points with N(0,1) targets, one
record then ten gradient passes", in fp64.  The metric is
trajectory-gradients/s over the whole step (record included); the gradient
pass alone is reported in config.grad_only_value.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--dtype f64|f32]
                  [--impl ours|reference] [--no-cpu-baseline] [--parity-sample K] [--no-secondary]

The lorenz_1m_solve workload times the adaptive forward-only solve instead
(gs_solve_adaptive on the same ensemble, no mesh kept; metric
trajectory-solves/s); lorenz_1m_sens times the forward sensitivities on the
recorded mesh (gs_sens: the sensitivity matrices at the ten save points and
the loss gradient; metric trajectory-sensitivities/s).

N > 1 runs under torchrun, one process per GPU; every rank owns its own
ensemble of the workload's size (weak scaling, no data-path collective:
trajectories are independent); timings are the max over ranks.  Inputs of the
default workload (mesh ~5 GB, checkpoints ~14 GB per rank) are far larger than
L2, so no flush is needed.  The CPU oracle appears twice: as ``cpu_baseline``
(a bounded sample timed on the host cores, rank 0, N = 1) and as the whole
``--impl reference`` arm.

The default run (lorenz_1m, fp64, full size, one process) also runs every
other workload briefly, each in a process of its own (3 warm-up + 3 timed
steps), and attaches their figures, or the error that stopped one, to its line
under ``secondary``.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# Peaks derived from unit counts and the maximum SM clock: 148 SMs x 64 FP64
# (128 FP32) fused multiply-adds per clock x 2 flops x 1965 MHz.
FP64_PEAK = 148 * 64 * 2 * 1965e6
FP32_PEAK = 148 * 128 * 2 * 1965e6

# Per workload: gradient passes per recorded mesh, algorithmic flops of one
# replay step (the forward step + its transposed step; fma = 2, division and
# tanh = 1), flops per save point (loss term + its gradient), the gradient
# kernel, and the configuration.
WORKLOADS = {
    "lorenz_1m": dict(passes=10, flop_step=192 + 264, flop_save=18, kernel="k_grad_tsit5_lorenz", n=1 << 20,
                      dtype="f64",
                      desc="Lorenz d=3, t in [0,10], Tsit5 rtol=atol=1e-6, 10 save points with N(0,1) targets, "
                           "1 record + 10 gradient passes"),
    # the headline with dense-output save points: steps stop only at t1, each
    # save time is read off Tsit5's continuous extension over its step's
    # stages (per save point: the weights and the combination 82 flop, the
    # transposed chain through the seven stages 281)
    "lorenz_1m_dense": dict(passes=10, flop_step=192 + 264, flop_save=18 + 82 + 281, kernel="k_grad_tsit5_lorenz",
                            problem="lorenz_1m", dense=True, n=1 << 20, dtype="f64",
                            desc="Lorenz d=3, t in [0,10], Tsit5 rtol=atol=1e-6, dense record (steps do not stop at "
                                 "the 10 save points; Tsit5's continuous extension there) with N(0,1) targets, "
                                 "1 record + 10 gradient passes"),
    # Verner's 7(6) pair on the headline ensemble and tolerance: the replay
    # step 321 (18 add, 45 mul, 129 fma: oracle count) + the transposed step
    # 420 (hand count: the nu combinations over the 30 nonzero a_mj and 7
    # weights b_j 222, nine Lorenz VJPs of 19 flop 171, the sum into lambda 27)
    "lorenz_1m_vern7": dict(passes=10, flop_step=321 + 420, flop_save=18, kernel="k_grad_vern7_lorenz",
                            problem="lorenz_1m", method="vern7", n=1 << 20, dtype="f64",
                            desc="Lorenz d=3, t in [0,10], Verner 7(6) rtol=atol=1e-6, 10 save points with N(0,1) "
                                 "targets, 1 record + 10 gradient passes"),
    "lorenz_small": dict(passes=1, flop_step=192 + 264, flop_save=12, kernel="k_grad_tsit5_lorenz", n=1024,
                         dtype="f64",
                         desc="Lorenz d=3, t in [0,1], Tsit5 rtol=atol=1e-8, loss sum ||u(T)||^2, "
                              "1 record + 1 gradient pass"),
    "robertson": dict(passes=1, flop_step=113 + 131, flop_save=9, kernel="k_grad_ros2", n=65536, dtype="f64",
                      desc="Robertson d=3, t in [0,1e5], ROS2 gamma=1+1/sqrt2, rtol=1e-6 atol=1e-10, "
                           "loss w . u(T), 1 record + 1 gradient pass"),
    # third-order Rosenbrock: the forward step 142 (7 add, 26 mul, 53 fma, 3
    # divisions, oracle count) + the transposed step 177 (hand count: three
    # transposed LU solves, two Robertson VJPs, the second-derivative term)
    "robertson_ros3": dict(passes=1, flop_step=142 + 177, flop_save=9, kernel="k_grad_ros3", problem="robertson",
                           method="ros3", n=65536, dtype="f64",
                           desc="Robertson d=3, t in [0,1e5], ROS3 (Sandu et al. 1997, order 3), rtol=1e-6 "
                                "atol=1e-10, loss w . u(T), 1 record + 1 gradient pass"),
    # the Rosenbrock path at d = 8 (kin8, 8 x 8 LU per step): the forward ROS3
    # step 966 (26 add, 76 mul, 428 fma, 8 divisions: oracle count of the dense
    # LU, its solves and the stages) + the transposed step 702 (hand count:
    # three transposed LU solves 360, two kin8 VJPs 108, the second-derivative
    # term 128, the stage combinations 106)
    "kin8": dict(passes=1, flop_step=966 + 702, flop_save=32, kernel="k_grad_kin8", n=262144, dtype="f64",
                 desc="kin8 d=8 stiff mass-action network (HIRES-sized ensemble), t in [0,100], ROS3 "
                      "rtol=atol=1e-7, loss sum ||u(T)||^2, 1 record + 1 gradient pass"),
    # the same with ROS2 (the configuration's second-order method): ~16,000
    # steps per trajectory at this tolerance, so a quarter of the ensemble
    # (checkpoints ~67 GB); forward step 807 (26 add, 77 mul, 348 fma, 8
    # divisions, oracle count) + transposed step 503 (hand count: two
    # transposed LU solves 240, two VJPs 108, second-derivative term 97,
    # combinations 58)
    "kin8_ros2": dict(passes=1, flop_step=807 + 503, flop_save=32, kernel="k_grad_kin8", problem="kin8",
                      method="ros2", n=65536, dtype="f64", smax=20000,
                      desc="kin8 d=8 stiff mass-action network, t in [0,100], ROS2 gamma=1+1/sqrt2 "
                           "rtol=atol=1e-7, loss sum ||u(T)||^2, 1 record + 1 gradient pass"),
    "node64": dict(passes=1, flop_step=52992 + 104076, flop_save=384, kernel="k_replay_node64", n=131072,
                   dtype="f32",
                   desc="du/dt = tanh(W u + b_i) - u, d=64, shared W, t in [0,1], Tsit5 rtol=atol=1e-5, "
                        "loss sum ||u(T)||^2, 1 record + 1 gradient pass"),
    # adaptive forward-only solve: flops per attempted step = the Tsit5 step
    # (192) + its error estimate (7-term combination, scaling, RMS norm: 56);
    # the step-size controller's scalar arithmetic is not counted
    "lorenz_1m_solve": dict(kind="solve", problem="lorenz_1m", flop_attempt=192 + 56, kernel="k_record3", n=1 << 20,
                            dtype="f64",
                            desc="Lorenz d=3, t in [0,10], Tsit5 rtol=atol=1e-6, states at 10 save points, "
                                 "one adaptive forward-only solve per step (no mesh kept)"),
    # forward sensitivities on the recorded mesh: flops per replay step = the
    # state (192) + 6 input directions x (tangent stage combinations 144 +
    # six Jacobian-vector products 108); the per-thread copies of the state
    # (one per direction) are not counted
    # forward sensitivities of the ROS3 replay on the robertson ensemble: the
    # state (142) + 6 directions x the tangent step (207: two JVPs, three
    # directional Jacobian products dJ k, three solves, the combinations; hand
    # count); the per-direction copies of the state are not counted
    "robertson_ros3_sens": dict(kind="sens", problem="robertson", method="ros3", flop_step=142 + 6 * 207,
                                kernel="k_sens_ros", n=65536, dtype="f64",
                                desc="Robertson d=3, t in [0,1e5], ROS3, rtol=1e-6 atol=1e-10, loss w . u(T); one "
                                     "forward-sensitivity pass per step on the recorded mesh (d u(T)/d(p,u0) + the "
                                     "loss gradient)"),
    # forward sensitivities with Verner's 7(6) pair: the state (321) + 6
    # directions x the tangent step (411: stage sums 204, u' 45, nine
    # Jacobian-vector products 162; hand count)
    "lorenz_1m_vern7_sens": dict(kind="sens", problem="lorenz_1m", method="vern7", flop_step=321 + 6 * 411,
                                 kernel="k_sens_vern7_lorenz", n=1 << 20, dtype="f64",
                                 desc="Lorenz d=3, t in [0,10], Verner 7(6) rtol=atol=1e-6, 10 save points with N(0,1) "
                                      "targets; one forward-sensitivity pass per step on the recorded mesh"),
    "lorenz_1m_sens": dict(kind="sens", problem="lorenz_1m", flop_step=192 + 6 * 252, kernel="k_sens_tsit5_lorenz",
                           n=1 << 20, dtype="f64",
                           desc="Lorenz d=3, t in [0,10], Tsit5 rtol=atol=1e-6, 10 save points with N(0,1) targets; "
                                "one forward-sensitivity pass per step on the recorded mesh (d u(t_k)/d(p,u0) at "
                                "every save point + the loss gradient)"),
}
# profile of the headline kernel (DRAM traffic per replay step), valid while
# the kernel's sources are unchanged
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "k_grad_tsit5_lorenz_traffic.json")
KERNEL_SOURCES = ["discrete_adjoint_b200/csrc/grad_tsit5.cu", "discrete_adjoint_b200/csrc/vec.cuh",
                  "discrete_adjoint_b200/csrc/common.cuh", "discrete_adjoint_b200/csrc/steps.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="lorenz_1m", choices=list(WORKLOADS))
    ap.add_argument("--dtype", default=None, choices=["f64", "f32"], help="default: the workload's own")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--n", type=int, default=None, help="trajectories per GPU (default: the workload's size)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parity-sample", type=int, default=0,
                    help="with --no-cpu-baseline: still report gradient parity on this many trajectories")
    ap.add_argument("--record", default="inplace", choices=["inplace", "full"],
                    help="per-step record: re-record in the setup record's slot order (gs_record_inplace), or "
                         "gs_record with its sort and gather")
    ap.add_argument("--no-secondary", action="store_true",
                    help="default run: skip the short runs of the other workloads")
    ap.add_argument("--products", default="tensor", choices=["simt", "tensor"],
                    help="d = 64 stage products: FP32 SIMT or tcgen05 3xTF32 (node64 only)")
    a = ap.parse_args()
    a.dtype = a.dtype or WORKLOADS[a.workload]["dtype"]
    a.n = a.n or WORKLOADS[a.workload]["n"]
    return a


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def distributed() -> bool:
    """Launched by torchrun (any world size, one included): the NCCL process
    group, its barriers and the max-over-ranks reductions run."""
    return "TORCHELASTIC_RUN_ID" in os.environ or int(os.environ.get("WORLD_SIZE", 1)) > 1


def metric_name(args) -> str:
    if args.workload == "lorenz_1m_dense":
        return f"trajectory-gradients/s (Lorenz {args.dtype.replace('f', 'fp')}, 1M traj, dense save points)"
    if args.workload == "lorenz_1m_vern7":
        return f"trajectory-gradients/s (Lorenz {args.dtype.replace('f', 'fp')}, 1M traj, Verner 7(6))"
    if args.workload == "lorenz_1m_vern7_sens":
        return f"trajectory-sensitivities/s (Lorenz Verner 7(6) {args.dtype.replace('f', 'fp')}, forward mode)"
    if args.workload == "lorenz_1m_sens":
        return f"trajectory-sensitivities/s (Lorenz {args.dtype.replace('f', 'fp')}, 1M traj, forward mode)"
    if args.workload == "robertson_ros3_sens":
        return f"trajectory-sensitivities/s (Robertson ROS3 {args.dtype.replace('f', 'fp')}, forward mode)"
    if args.workload == "lorenz_1m_solve":
        return f"trajectory-solves/s (Lorenz {args.dtype.replace('f', 'fp')}, 1M traj, adaptive forward-only)"
    if args.workload == "lorenz_1m":
        return f"trajectory-gradients/s (Lorenz {args.dtype.replace('f', 'fp')}, 1M traj)"
    return f"trajectory-gradients/s ({args.workload} {args.dtype.replace('f', 'fp')})"


def make_problem(args, seed_offset=0, n=None):
    import workloads
    name = WORKLOADS[args.workload].get("problem", args.workload)
    prob = workloads.by_name(name, n=n or args.n, dtype=args.dtype, seed_offset=seed_offset)
    if "method" in WORKLOADS[args.workload]:
        prob.method = WORKLOADS[args.workload]["method"]
    return prob


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"gs_clocks_{os.getpid()}.csv")
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


def smax_cap(workload):
    import workloads
    W = WORKLOADS[workload]
    return W.get("smax") or 4 * workloads.SMAX[W.get("problem", workload)]


def oracle_step_time(prob, threads, passes, cap, dense=False):
    """Oracle record (step capacity `cap`) + `passes` tape gradient passes of
    `prob` on the host."""
    import oracle
    t0 = time.perf_counter()
    om = oracle.record(prob, cap, nthreads=threads, dense=dense)
    t1 = time.perf_counter()
    oracle.grad(prob, om, nthreads=threads)
    t2 = time.perf_counter()
    return t1 - t0, t2 - t1, (t1 - t0) + passes * (t2 - t1)


def cpu_baseline(args, sample: int):
    """The oracle as it stands: record + one gradient pass of a sample of the
    workload on the host cores, scaled to the step's record + passes (the
    solve workload: the oracle's adaptive solve of the sample)."""
    import oracle
    prob = make_problem(args).subset(np.arange(sample))
    threads = oracle.default_threads()
    if WORKLOADS[args.workload].get("kind") == "solve":
        t0 = time.perf_counter()
        oracle.solve_adaptive(prob, smax_cap(args.workload), nthreads=threads)
        dt = time.perf_counter() - t0
        return {"value": sample / dt, "unit": "trajectory-solves/s", "cores": threads, "kind": "oracle",
                "sample": f"first {sample} of the {args.n} trajectories: oracle adaptive solve {dt:.2f} s"}
    if WORKLOADS[args.workload].get("kind") == "sens":
        om = oracle.record(prob, smax_cap(args.workload), nthreads=threads)
        t0 = time.perf_counter()
        oracle.sens(prob, om, nthreads=threads)
        dt = time.perf_counter() - t0
        return {"value": sample / dt, "unit": "trajectory-sensitivities/s", "cores": threads, "kind": "oracle",
                "sample": f"first {sample} of the {args.n} trajectories on the oracle's own mesh: dual-number "
                          f"sensitivities {dt:.2f} s"}
    passes = WORKLOADS[args.workload]["passes"]
    tr, tg, per_step = oracle_step_time(prob, threads, passes, smax_cap(args.workload),
                                        WORKLOADS[args.workload].get("dense", False))
    return {"value": sample * passes / per_step, "unit": "trajectory-gradients/s", "cores": threads,
            "kind": "oracle",
            "sample": f"first {sample} of the {args.n} trajectories: oracle record {tr:.2f} s + one tape gradient "
                      f"pass {tg:.2f} s, scaled to 1 record + {passes} passes"}


def parity_sample(args, sample: int):
    """Gradient parity of the GPU kernel on a sample of the workload, in the
    step's launch configuration: the oracle records the sample, the library's
    gs_grad runs on that mesh (slot j = trajectory j), and each trajectory's
    error is ||g - g_ref||_inf / ||g_ref||_inf over (dp, du0) against the
    oracle's tape with its reverse sweep accumulated in extended precision.
    The oracle's own plain-precision tape error on the same sample is reported
    beside it: on chaotic trajectories the reverse sweep's conditioning puts
    both near the gate."""
    import torch

    import oracle
    import discrete_adjoint_b200 as gs
    W = WORKLOADS[args.workload]
    prob = make_problem(args).subset(np.arange(sample))
    threads = oracle.default_threads()
    om = oracle.record(prob, smax_cap(args.workload), nthreads=threads, dense=W.get("dense", False))
    dev = torch.device("cuda", torch.cuda.current_device())
    td = torch.float64 if args.dtype == "f64" else torch.float32
    f = lambda a: torch.tensor(np.ascontiguousarray(a), dtype=td, device=dev)
    i32 = lambda a: torch.tensor(np.ascontiguousarray(a, dtype=np.int32), device=dev)
    ens = gs.Ensemble(prob.system, prob.method, args.dtype, f(prob.p), f(prob.u0), prob.t0, prob.t1,
                      [float(x) for x in prob.tsave], None if prob.W is None else f(prob.W))
    mesh = gs.Mesh(f(om.h.T), i32(np.arange(sample)), i32(om.nsteps), i32(om.save_idx.T), i32(om.status),
                   i32(om.nreject), None if om.theta is None else f(om.theta.T))
    out = gs.gs_grad(ens, mesh, loss=prob.loss, target=None if prob.target is None else f(prob.target),
                     weight=None if prob.weight is None else f(prob.weight))
    torch.cuda.synchronize()
    g = np.vstack([out.dp.double().cpu().numpy(), out.du0.double().cpu().numpy()])
    wide = oracle.grad(prob, om, "tape_wide", nthreads=threads)
    r = np.vstack([wide["dp"], wide["du0"]])
    ok = om.status == 0
    rel = lambda a: (np.abs(a - r).max(0) / np.abs(r).max(0))[ok]
    e = rel(g)
    # kappa_i: the largest error of the oracle's own routes in the kernel's
    # precision (its tape, the tape with fused adjoint updates, its dual
    # numbers where built) on trajectory i
    routes = ("tape", "tape_fused") + (("dual",) if prob.system != "node64" else ())
    errs = {m: rel(np.vstack([(o := oracle.grad(prob, om, m, nthreads=threads))["dp"], o["du0"]]))
            for m in routes}
    k = np.max(np.vstack(list(errs.values())), axis=0)
    gate = 1e-12 if args.dtype == "f64" else 1e-4
    bound = np.maximum(gate, 4.0 * k)
    q = lambda a, x: float(np.quantile(a, x)) if len(a) else None
    return {"sample": f"first {sample} trajectories, oracle mesh", "reference": "oracle tape, extended-precision "
            "reverse sweep", "metric": "per-trajectory ||g - g_ref||_inf / ||g_ref||_inf over (dp, du0)",
            "p50": q(e, 0.5), "p99": q(e, 0.99), "max": q(e, 1.0), "gate": gate,
            "frac_within_gate": float(np.mean(e <= gate)) if len(e) else None,
            "rule": "e_i <= max(gate, 4 kappa_i), kappa_i = largest error of the oracle's own routes "
                    "(%s) in this precision on trajectory i" % ", ".join(routes),
            "frac_within_rule": float(np.mean(e <= bound)) if len(e) else None,
            "max_over_rule": float(np.max(e / bound)) if len(e) else None,
            "oracle_tape": {"p50": q(errs["tape"], 0.5), "p99": q(errs["tape"], 0.99), "max": q(errs["tape"], 1.0)}}


def run_reference(args):
    """--impl reference: the CPU oracle on the host cores, same metric/config;
    each step is the record + gradient passes of a bounded sample."""
    import oracle
    rank, world, _ = dist_env()
    if rank != 0:
        return
    W = WORKLOADS[args.workload]
    kind = W.get("kind", "grad")
    solve = kind != "grad"
    sample = {"lorenz_1m": 256, "lorenz_1m_dense": 256, "lorenz_1m_vern7": 256, "lorenz_small": 256,
              "robertson": 32, "node64": 64,
              "lorenz_1m_solve": 4096, "lorenz_1m_sens": 512, "lorenz_1m_vern7_sens": 512, "robertson_ros3": 256,
              "robertson_ros3_sens": 256, "kin8": 256, "kin8_ros2": 16}[args.workload]
    prob = make_problem(args).subset(np.arange(sample))
    threads = oracle.default_threads()
    om = oracle.record(prob, smax_cap(args.workload), nthreads=threads) if kind == "sens" else None
    times = []
    for it in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        if kind == "solve":
            oracle.solve_adaptive(prob, smax_cap(args.workload), nthreads=threads)
        elif kind == "sens":
            oracle.sens(prob, om, nthreads=threads)
        else:
            om = oracle.record(prob, smax_cap(args.workload), nthreads=threads, dense=W.get("dense", False))
            for _ in range(W["passes"]):
                oracle.grad(prob, om, nthreads=threads)
        dt = time.perf_counter() - t0
        if it >= args.warmup:
            times.append(dt)
    t = float(np.mean(times))
    passes = 1 if solve else W["passes"]
    unit = {"solve": "trajectory-solves/s", "sens": "trajectory-sensitivities/s"}.get(kind, "trajectory-gradients/s")
    what = {"solve": "oracle adaptive solve", "sens": "oracle dual-number sensitivities on its own mesh"}.get(kind)
    what = what or f"oracle record + {W['passes']} tape gradient passes"
    value = sample * passes / t
    line = {"impl": "reference", "metric": metric_name(args), "value": value, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.dtype,
            "data": "synthetic",
            "config": {"workload": f"{args.workload}: {W['desc']}; n={args.n} per GPU",
                       "sample_per_step": sample},
            "cpu_baseline": {"value": value, "unit": unit, "cores": threads, "kind": "oracle",
                             "sample": f"first {sample} trajectories per step ({what})"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def kernel_traffic(total_steps: int):
    """DRAM bytes per gradient launch from the committed ncu capture, scaled by
    replay steps, or None if the kernel changed since the capture."""
    try:
        prof = json.load(open(TRAFFIC_FILE))
        h = hashlib.sha256()
        for f in KERNEL_SOURCES:
            h.update(open(os.path.join(ROOT, f), "rb").read())
        if h.hexdigest() != prof["sources_sha256"]:
            return None
        return prof["dram_bytes"] / prof["replay_steps"] * total_steps
    except Exception:
        return None


def run_single(args):
    """One library call per step over the rank's ensemble: the adaptive
    forward-only solve (gs_solve_adaptive) or the forward sensitivities on the
    recorded mesh (gs_sens)."""
    import torch
    import torch.distributed as dist

    import discrete_adjoint_b200 as gs

    W = WORKLOADS[args.workload]
    kind = W["kind"]
    rank, world, local = dist_env()
    dist_on = distributed()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if dist_on:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    n = args.n
    prob = make_problem(args, seed_offset=rank)
    td = torch.float64 if args.dtype == "f64" else torch.float32
    esz = 8 if args.dtype == "f64" else 4
    stream = torch.cuda.current_stream()
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(td).pin_memory()
    host = {"p": pin(prob.p), "u0": pin(prob.u0)}
    if kind == "sens" and prob.target is not None:
        host["target"] = pin(prob.target)
    if kind == "sens" and prob.weight is not None:
        host["weight"] = pin(prob.weight)
    d = {k: v.to(dev) for k, v in host.items()}
    ens = gs.Ensemble(prob.system, prob.method, args.dtype, d["p"], d["u0"], prob.t0, prob.t1,
                      [float(x) for x in prob.tsave])
    smax = smax_cap(args.workload)
    # setup (untimed): a record, for the attempted-step count of the solve's
    # flop figure or as the mesh the sensitivities run on
    nst, _ = gs.gs_count(ens, prob.rtol, prob.atol, smax)
    mesh = gs.new_mesh(n, int(nst.max().item()), len(prob.tsave), args.dtype, dev)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol, stream=stream)
    accepted = mesh.nsteps.double()
    if kind == "solve":
        attempts = int(mesh.nsteps.sum().item() + mesh.nreject.sum().item())
        flops = W["flop_attempt"] * attempts
        # the solves run in the setup record's slot order (trajectories of
        # equal step count side by side in a warp); --record full: in
        # trajectory order (gs_solve_adaptive)
        order = mesh.order.clone()
        del mesh
        u_save = torch.empty((len(prob.tsave), prob.d, n), dtype=td, device=dev)
        nsteps = torch.empty(n, dtype=torch.int32, device=dev)
        status = torch.empty(n, dtype=torch.int32, device=dev)
        ws_solve = gs.workspace(gs.gradsolve.RECORD_INPLACE_WS, dev)
        outputs = [u_save]
        ordered = args.record == "inplace"
        work = {"attempted_steps": attempts,
                "solve": ("gs_solve_adaptive_ordered in the slot order of a setup record of the ensemble"
                          if ordered else "gs_solve_adaptive in trajectory order")}

        def step():
            if ordered:
                gs.gs_solve_adaptive_ordered(ens, prob.rtol, prob.atol, smax, order, u_save=u_save, nsteps=nsteps,
                                             status=status, ws=ws_solve, stream=stream)
            else:
                gs.gs_solve_adaptive(ens, prob.rtol, prob.atol, smax, u_save=u_save, nsteps=nsteps, status=status,
                                     stream=stream)
    else:
        total_steps = int(mesh.nsteps.sum().item())
        flops = W["flop_step"] * total_steps
        out = gs.new_grad_out(ens)
        sens = torch.empty((len(prob.tsave), prob.d, prob.np_ + prob.d, n), dtype=td, device=dev)
        outputs = [sens, out.loss, out.dp, out.du0]
        status = mesh.status
        work = {"replay_steps": total_steps, "sens_gb": sens.numel() * esz / 1e9}

        def step():
            gs.gs_sens(ens, mesh, loss=prob.loss, target=d.get("target"), weight=d.get("weight"), out=out, sens=sens,
                       stream=stream)

    # what the timed loop streams (the mesh for the sensitivities, the outputs
    # for the solve) against the 126 MB L2: larger means no flush is needed
    out_gb = sum(t.numel() * t.element_size() for t in outputs) / 1e9
    mesh_gb = mesh.h.numel() * esz / 1e9 if kind == "sens" else 0.0
    big = max(out_gb, mesh_gb) > 0.126
    l2_note = "mesh %.2f GB, outputs %.2f GB: %s" % (
        mesh_gb, out_gb, "larger than L2, no flush" if big else "fits in L2 (compute-bound kernel), no flush")

    def barrier():
        if dist_on:
            dist.barrier()
        torch.cuda.synchronize()

    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(args.warmup):
        step()
    barrier()
    clk = ClockSampler(bus_id_of(dev))
    launches0 = gs.gs_launch_count()
    barrier()
    t_start, t_end = ev(), ev()
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_end.record(stream)
    barrier()
    launches = gs.gs_launch_count() - launches0
    clocks = clk.stop()
    tmax = torch.tensor([t_start.elapsed_time(t_end) / 1e3], dtype=torch.float64, device=dev)
    if dist_on:
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
    elapsed = float(tmax.item())
    assert (status == 0).all()

    # end to end from host buffers: H2D of the inputs, the call, D2H of its results
    h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outputs]

    def e2e_step():
        for k, v in host.items():
            d[k].copy_(v, non_blocking=True)
        step()
        for hb, t in zip(h_out, outputs):
            hb.copy_(t, non_blocking=True)

    e2e_step()
    barrier()
    e2e_steps = max(1, min(args.steps, 3))
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    barrier()
    e2e_t = torch.tensor([a.elapsed_time(b) / 1e3 / e2e_steps], dtype=torch.float64, device=dev)
    if dist_on:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)

    unit = "trajectory-solves/s" if kind == "solve" else "trajectory-sensitivities/s"
    t_call = elapsed / args.steps
    achieved = flops / t_call
    peak = FP64_PEAK if args.dtype == "f64" else FP32_PEAK
    line = {
        "metric": metric_name(args), "value": world * n * args.steps / elapsed, "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_call * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": dict({"workload": f"{args.workload}: {W['desc']}; n={n} per GPU", "n_per_gpu": n,
                        "steps_mean": float(accepted.mean()),
                        "steps_max_over_mean": float(accepted.max() / accepted.mean()),
                        "l2": l2_note,
                        "parallelism": f"dp{world} (independent trajectory shards)"}, **work),
        "clocks": clocks,
        "e2e": {"value": world * n / float(e2e_t.item()), "unit": unit,
                "h2d_bytes_per_step": sum(v.numel() for v in host.values()) * esz,
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in h_out)},
        "gpu_launches": launches,
        "roofline": {"bound": "alu", "achieved": achieved / 1e12, "peak": peak / 1e12, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None, "kernel": W["kernel"],
                     "peak_source": "derived: 148 SMs x %d %s FMA/clk x 2 x 1965 MHz" % (
                         64 if args.dtype == "f64" else 128, "FP64" if args.dtype == "f64" else "FP32"),
                     "flops_per_launch": flops},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args, min(262144 if kind == "solve" else 32768, n))
    if dist_on:
        dist.barrier()
        dist.destroy_process_group()
    return line if rank == 0 else None


def tensor_roofline(alu, total_steps, grad_ms):
    """Roofline of the d = 64 gradient with its products on the tensor cores:
    the algorithmic product work (forward W U: 6, transposed step W^T g and
    g U^T: 12 products of 64 x 64 per replay step, 2 flops per multiply-add,
    fp32 accuracy) against the TF32 dense peak, taken as the measured bf16
    GEMM peak (MEASURED_PEAKS.json, burst) times the nominal TF32 / bf16 ratio
    1.1 / 2.25.  The 3xTF32 split issues three TF32 products per fp32 one;
    those are implementation, not algorithmic work.  The ALU form (all
    algorithmic flops against the FP32 peak) is kept beside it."""
    gemm = 18 * 64 * 64 * 2 * total_steps
    try:
        bf16 = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"] * 1e12
        src = "measured bf16 %.1f TF/s x 1.1/2.25 (nominal TF32/bf16)" % (bf16 / 1e12)
    except Exception:
        bf16 = 1.59e15
        src = "fallback bf16 1590 TF/s x 1.1/2.25 (nominal TF32/bf16)"
    peak = bf16 * 1.1 / 2.25
    achieved = gemm / (grad_ms / 1e3)
    return {"bound": "tensor", "achieved": achieved / 1e12, "peak": peak / 1e12, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": None, "kernel": "k_node64_t128", "peak_source": src,
            "flops_per_launch": gemm, "alu": {k: alu[k] for k in ("achieved", "peak", "frac", "flops_per_launch")}}


def run_ours(args):
    import torch
    import torch.distributed as dist

    import discrete_adjoint_b200 as gs

    W = WORKLOADS[args.workload]
    passes = W["passes"]
    rank, world, local = dist_env()
    dist_on = distributed()
    torch.cuda.set_device(local)
    gs.gs_set_option(gs.gradsolve.OPT_NODE64_TENSOR_CORES, int(args.products == "tensor"))
    dev = torch.device("cuda", local)
    if dist_on:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    n = args.n
    prob = make_problem(args, seed_offset=rank)
    td = torch.float64 if args.dtype == "f64" else torch.float32
    esz = 8 if args.dtype == "f64" else 4
    stream = torch.cuda.current_stream()

    # host inputs (pinned) and their device copies
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(td).pin_memory()
    host = {"p": pin(prob.p), "u0": pin(prob.u0)}
    if prob.target is not None:
        host["target"] = pin(prob.target)
    if prob.weight is not None:
        host["weight"] = pin(prob.weight)
    if prob.W is not None:
        host["W"] = pin(prob.W)
    d = {k: v.to(dev) for k, v in host.items()}
    ens = gs.Ensemble(prob.system, prob.method, args.dtype, d["p"], d["u0"], prob.t0, prob.t1,
                      [float(x) for x in prob.tsave], d.get("W"))
    loss_kw = dict(loss=prob.loss, target=d.get("target"), weight=d.get("weight"))

    # sizing pass (setup, untimed): mesh capacity = the longest chain
    dense = W.get("dense", False)
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, smax_cap(args.workload), dense=dense, stream=stream)
    smax = int(nsteps.max().item())
    # its time, on a second call (the first also loads the library's kernels)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    gs.gs_count(ens, prob.rtol, prob.atol, smax_cap(args.workload), nsteps=nsteps, dense=dense, stream=stream)
    c1.record(stream)
    c1.synchronize()
    count_ms = c0.elapsed_time(c1)
    mesh = gs.new_mesh(n, smax, len(prob.tsave), args.dtype, dev, dense=dense)
    ws_rec = gs.workspace(gs.gs_workspace_bytes(ens, mesh, gs.gradsolve.OP_RECORD), dev)
    ws_grad = gs.workspace(gs.gs_workspace_bytes(ens, mesh, gs.gradsolve.OP_GRAD), dev)
    outs = [gs.new_grad_out(ens) for _ in range(2)]

    ev = lambda: torch.cuda.Event(enable_timing=True)
    grad_events, rec_events = [], []
    # The first record of the ensemble (setup, untimed): gs_record sorts the
    # slots by step count and gathers the mesh into that order.  The steps then
    # re-record the ensemble in that slot order (gs_record_inplace: straight
    # into the mesh, no sort or gather), as a loop that re-records one ensemble
    # does; --record full runs gs_record in every step instead.
    inplace = args.record == "inplace" and prob.system != "node64"
    f0, f1 = ev(), ev()
    gs.gs_record(ens, mesh, prob.rtol, prob.atol, ws=ws_rec, stream=stream)
    f0.record(stream)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol, ws=ws_rec, stream=stream)
    f1.record(stream)
    f1.synchronize()
    full_record_ms = f0.elapsed_time(f1)

    def record():
        if inplace:
            gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol, ws=ws_rec, stream=stream)
        else:
            gs.gs_record(ens, mesh, prob.rtol, prob.atol, ws=ws_rec, stream=stream)

    def step(timing):
        if timing:
            e0 = ev()
            e0.record(stream)
        record()
        if timing:
            e1 = ev()
            e1.record(stream)
            rec_events.append((e0, e1))
        for k in range(passes):
            if timing:
                a = ev()
                a.record(stream)
            gs.gs_grad(ens, mesh, out=outs[k % 2], ws=ws_grad, stream=stream, **loss_kw)
            if timing:
                b = ev()
                b.record(stream)
                grad_events.append((a, b))

    def barrier():
        if dist_on:
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
    if dist_on:
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
    elapsed, grad_ms, rec_ms = tmax.tolist()

    # End to end through the public API from host buffers: H2D of the inputs,
    # the record, and per pass the gradient plus a D2H read of its results.
    # Pass k's results go back on a copy stream while pass k + 1 computes into
    # the other output buffer (the compute stream waits before reusing one).
    o0 = outs[0]
    shapes = [t.shape for t in (o0.loss, o0.dp, o0.du0)] + ([o0.dshared.shape] if o0.dshared is not None else [])
    h_out = [[torch.empty(sh, dtype=td).pin_memory() for sh in shapes] for _ in range(2)]
    copy_stream = torch.cuda.Stream(device=dev)
    done_copy = [torch.cuda.Event(), torch.cuda.Event()]
    done_grad = [torch.cuda.Event(), torch.cuda.Event()]

    # the record needs p, u0 (and W); the targets and weights are needed from
    # the first gradient pass on, so they cross on the copy stream while the
    # record runs (after the previous step's passes are done with them)
    side = [k for k in host if k in ("target", "weight")]
    side_ready = torch.cuda.Event()

    def e2e_step():
        for k, v in host.items():
            if k not in side:
                d[k].copy_(v, non_blocking=True)
        if side:
            copy_stream.wait_stream(stream)
            with torch.cuda.stream(copy_stream):
                for k in side:
                    d[k].copy_(host[k], non_blocking=True)
            side_ready.record(copy_stream)
        record()
        if side:
            stream.wait_event(side_ready)
        for k in range(passes):
            b = k % 2
            o = outs[b]
            stream.wait_event(done_copy[b])  # its previous contents are on the host
            gs.gs_grad(ens, mesh, out=o, ws=ws_grad, stream=stream, **loss_kw)
            done_grad[b].record(stream)
            copy_stream.wait_event(done_grad[b])
            with torch.cuda.stream(copy_stream):
                srcs = [o.loss, o.dp, o.du0] + ([o.dshared] if o.dshared is not None else [])
                for hb, src in zip(h_out[b], srcs):
                    hb.copy_(src, non_blocking=True)
            done_copy[b].record(copy_stream)
        stream.wait_stream(copy_stream)

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
    if dist_on:
        dist.all_reduce(e2e_t, op=dist.ReduceOp.MAX)
    h2d = sum(v.numel() for v in host.values()) * esz
    d2h = passes * sum(t.numel() for t in h_out[0]) * esz

    # algorithmic work of one gradient launch
    total_steps = int(mesh.nsteps.sum().item())
    flops = W["flop_step"] * total_steps + W["flop_save"] * len(prob.tsave) * n
    achieved = flops / (grad_ms / 1e3)
    peak = FP64_PEAK if args.dtype == "f64" else FP32_PEAK
    ns = mesh.nsteps.double()
    value = world * n * passes * args.steps / elapsed
    traffic = kernel_traffic(total_steps) if (args.workload == "lorenz_1m" and args.dtype == "f64") else None
    line = {
        "metric": metric_name(args), "value": value, "unit": "trajectory-gradients/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": args.dtype, "data": "synthetic",
        "config": {"workload": f"{args.workload}: {W['desc']}; n={n} per GPU",
                   "n_per_gpu": n, "passes_per_step": passes, "smax": smax,
                   "steps_total": total_steps, "steps_mean": float(ns.mean()),
                   "steps_max_over_mean": float(ns.max() / ns.mean()),
                   "rejects_total": int(mesh.nreject.sum().item()),
                   "grad_ms": grad_ms, "record_ms": rec_ms, "grad_only_value": world * n / (grad_ms / 1e3),
                   "count_ms": count_ms,
                   "count_note": "sizing pass (gs_count) run once as untimed setup; the timed records reuse the "
                                 "capacity it found",
                   "record": ("gs_record_inplace (the ensemble re-recorded in the slot order its setup record set, "
                              "straight into the mesh)" if inplace else "gs_record (adaptive pass, slot sort by step "
                              "count, gather into slot order)"),
                   "full_record_ms": full_record_ms,
                   "full_record_note": "gs_record with its sort and gather, timed once in setup",
                   "l2": "inputs larger than L2 (mesh %.2f GB, gradient workspace %.2f GB); no flush" % (
                       mesh.h.numel() * esz / 1e9, ws_grad.numel() / 1e9),
                   "parallelism": f"dp{world} (independent trajectory shards)",
                   **({"products": args.products} if args.workload == "node64" else {})},
        "clocks": clocks,
        "e2e": {"value": world * n * passes / float(e2e_t.item()), "unit": "trajectory-gradients/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        "roofline": {"bound": "alu", "achieved": achieved / 1e12, "peak": peak / 1e12, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "kernel": W["kernel"],
                     "peak_source": "derived: 148 SMs x %d %s FMA/clk x 2 x 1965 MHz" % (
                         64 if args.dtype == "f64" else 128, "FP64" if args.dtype == "f64" else "FP32"),
                     "flops_per_launch": flops},
    }
    if args.workload == "node64" and args.products == "tensor":
        line["roofline"] = tensor_roofline(line["roofline"], total_steps, grad_ms)
    elif clocks and clocks.get("sm_mhz"):
        # the same work against the peak at the median SM clock of the timed
        # region (the 1000 W cap lowers it under sustained FP64 load); the
        # headline fraction above stays against the maximum clock
        line["roofline"]["frac_at_sm_clock"] = line["roofline"]["frac"] * 1965.0 / clocks["sm_mhz"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # samples sized for seconds of host work (and host memory for the
        # oracle's trajectory-major meshes)
        sample = {"lorenz_1m": 32768, "lorenz_1m_dense": 32768, "lorenz_1m_vern7": 32768, "lorenz_small": 1024,
                  "robertson": 256,
                  "robertson_ros3": 2048, "node64": 1024, "kin8": 2048, "kin8_ros2": 64}[args.workload]
        line["cpu_baseline"] = cpu_baseline(args, min(sample, n))
        psample = {"lorenz_1m": 8192, "lorenz_1m_dense": 8192, "lorenz_1m_vern7": 8192, "lorenz_small": 1024,
                   "robertson": 256,
                   "robertson_ros3": 2048, "node64": 256, "kin8": 1024, "kin8_ros2": 32}[args.workload]
        line["parity"] = parity_sample(args, min(psample, n))
    elif rank == 0 and world == 1 and args.parity_sample:
        line["parity"] = parity_sample(args, min(args.parity_sample, n))
    if dist_on:
        dist.barrier()
        dist.destroy_process_group()
    return line if rank == 0 else None


# Short runs of the other workloads, attached to the default run's line: name,
# bench arguments, trajectories in its parity sample (0: none)
SECONDARY = [
    ("lorenz_1m_f32", ["--workload", "lorenz_1m", "--dtype", "f32"], 2048),
    ("lorenz_1m_dense", ["--workload", "lorenz_1m_dense"], 2048),
    ("lorenz_1m_vern7", ["--workload", "lorenz_1m_vern7"], 2048),
    ("robertson_ros2", ["--workload", "robertson"], 128),
    ("robertson_ros3", ["--workload", "robertson_ros3"], 512),
    ("kin8_ros3", ["--workload", "kin8"], 256),
    ("node64_tensor", ["--workload", "node64"], 128),
    ("lorenz_1m_solve", ["--workload", "lorenz_1m_solve"], 0),
    ("lorenz_1m_sens", ["--workload", "lorenz_1m_sens"], 0),
    ("lorenz_1m_vern7_sens", ["--workload", "lorenz_1m_vern7_sens"], 0),
    ("robertson_ros3_sens", ["--workload", "robertson_ros3_sens"], 0),
]


def wants_secondary(args) -> bool:
    return (args.impl == "ours" and not args.no_secondary and not distributed() and args.workload == "lorenz_1m"
            and args.dtype == "f64" and args.n == WORKLOADS["lorenz_1m"]["n"])


def run_secondary():
    """Each other workload at its full size in a process of its own (3 warm-up
    + 3 timed steps, no CPU baseline): the figures of its line that a reader
    compares, or the error that stopped it."""
    res = {}
    for name, extra, psample in SECONDARY:
        cmd = [sys.executable, os.path.abspath(__file__), *extra, "--steps", "3", "--warmup", "3",
               "--no-cpu-baseline", "--no-secondary"] + (["--parity-sample", str(psample)] if psample else [])
        try:
            r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
            js = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
            if r.returncode != 0 or not js:
                tail = (r.stderr or r.stdout).strip().splitlines()[-1:] or [""]
                res[name] = {"error": f"exit {r.returncode}: {tail[0][:300]}"}
                continue
            ln = json.loads(js[-1])
            cfg, rf = ln["config"], ln["roofline"]
            res[name] = {"workload": cfg["workload"], "metric": ln["metric"], "value": ln["value"],
                         "unit": ln["unit"], "dtype": ln["dtype"], "ms_per_step": ln["ms_per_step"],
                         "steps": ln["steps"], "warmup": ln["warmup"],
                         **{k: cfg[k] for k in ("grad_ms", "record_ms", "full_record_ms") if k in cfg},
                         "roofline": {k: rf.get(k) for k in ("bound", "kernel", "achieved", "peak", "unit", "frac",
                                                             "frac_at_sm_clock")},
                         "e2e": ln["e2e"]["value"], "clocks": ln["clocks"], "gpu_launches": ln["gpu_launches"],
                         **({"parity": ln["parity"]} if "parity" in ln else {})}
        except Exception as e:  # a secondary never takes the headline line down
            res[name] = {"error": f"{type(e).__name__}: {str(e)[:300]}"}
    return res


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    if WORKLOADS[args.workload].get("kind") in ("solve", "sens"):
        line = run_single(args)
    else:
        line = run_ours(args)
    if line is None:
        return
    if wants_secondary(args):
        import torch
        torch.cuda.empty_cache()
        line["secondary"] = run_secondary()
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
