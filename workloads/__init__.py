"""Seeded synthetic ensembles for the five benchmark workloads.

This module only draws random inputs and states the problem sizes; it holds
none of the method's arithmetic, so both the CUDA library's tests/bench and
the CPU oracle can take their inputs from it without sharing any of the method.

Workloads (GRADSOLVE, arXiv 2609.02876: the Lorenz and Robertson studies of
the evolve.pub review "Summary", the neural right-hand side named there as
well; the distributions are those of the benchmark configurations):

  lorenz_small  n=1,024   Lorenz, fp64, t in [0,1], rtol=atol=1e-8,
                loss = sum ||u(T)||^2.
  lorenz_1m     n=2**20   Lorenz, fp64 (fp32 variant: same draws rounded),
                t in [0,10], rtol=atol=1e-6, loss = sum over t_k = 1..10 of
                ||u(t_k) - target_k||^2 with target ~ N(0,1).
  robertson     n=65,536  Robertson kinetics, ROS2, fp64, t in [0,1e5],
                rtol=1e-6, atol=1e-10, loss = w . u(T), w ~ U[0,1]^3.
  hires         (not built: the HIRES equations and rate constants are not
                given by the sources this library follows)
  node64        n=131,072 du/dt = tanh(W u + b_i) - u, d=64, fp32, t in [0,1],
                rtol=atol=1e-5, loss = sum ||u(T)||^2.
  kin8          n=262,144, an 8-species stiff mass-action network defined
                by this library, d=8, np=8, ROS3, fp64, t in [0, 100],
                rtol=atol=1e-7, loss = sum ||u(T)||^2, rate constants spread
                by lognormal(0, 0.05): the Rosenbrock path at d=8 (8x8 LU),
                with HIRES's ensemble size, tolerances and loss (HIRES itself
                is not built).  Nominal rate constants
                k = (800, 400, 2, 0.2, 0.05, 0.025, 6, 0.004), each scaled by
                lognormal(0, 0.05); u0 = (1, 0, 0.5, 0, 0, 0, 0.3, 0).

Distribution notation: N(m, v) has VARIANCE v; lognormal(0, s) is exp(N(0, s^2))
(s is the standard deviation of the log); u0 = (1,0,0) + eps * (1,1,1) draws ONE
scalar eps ~ N(0, 0.01) per trajectory.

Layouts: structure-of-arrays, p [np][n], u0 [d][n], target/weight
[nsave][d][n], W [64][64] row-major.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

SEED_BASE = 20261201

CONFIG_INDEX = {"lorenz_small": 0, "lorenz_1m": 1, "robertson": 2, "hires": 3, "node64": 4, "kin8": 5}

FULL_N = {"lorenz_small": 1024, "lorenz_1m": 1 << 20, "robertson": 65536, "hires": 262144, "node64": 131072,
          "kin8": 262144}

# Recorded-step capacity each workload is sized for (the recorder reports
# MAXSTEPS beyond it); generous relative to the observed maxima.
SMAX = {"lorenz_small": 256, "lorenz_1m": 1024, "robertson": 8192, "node64": 256, "kin8": 2048}


@dataclass
class Problem:
    system: str            # "lorenz" | "robertson" | "node64" | "kin8" | "linear"
    method: str            # "tsit5" | "ros2" | "ros3"
    dtype: str             # "f64" | "f32"
    n: int
    d: int
    np_: int
    p: np.ndarray          # [np][n] float64 draws (rounded to fp32 for f32 runs)
    u0: np.ndarray         # [d][n]
    t0: float
    t1: float
    tsave: np.ndarray      # [nsave] float64, strictly increasing, in (t0, t1]
    rtol: float
    atol: float
    loss: str              # "sumsq" | "linear"
    target: np.ndarray | None = None   # [nsave][d][n] (sumsq; None = zero)
    weight: np.ndarray | None = None   # [nsave][d][n] (linear)
    W: np.ndarray | None = None        # [64][64] (node64)
    name: str = ""
    meta: dict = field(default_factory=dict)

    def subset(self, idx) -> "Problem":
        """The same problem restricted to trajectories ``idx`` (in that order)."""
        idx = np.asarray(idx)
        return replace(self, n=len(idx), p=self.p[:, idx].copy(), u0=self.u0[:, idx].copy(),
                       target=None if self.target is None else self.target[:, :, idx].copy(),
                       weight=None if self.weight is None else self.weight[:, :, idx].copy())

    def as_dtype(self, dtype: str) -> "Problem":
        """Same draws, arithmetic type ``dtype`` (inputs rounded for fp32)."""
        if dtype == "f64":
            return replace(self, dtype="f64")
        r = lambda a: None if a is None else a.astype(np.float32).astype(np.float64)
        return replace(self, dtype="f32", p=r(self.p), u0=r(self.u0), target=r(self.target),
                       weight=r(self.weight), W=r(self.W), tsave=r(self.tsave))


def _rng(name: str, seed_offset: int = 0):
    return np.random.default_rng(np.random.PCG64(SEED_BASE + CONFIG_INDEX[name] + 1000 * seed_offset))


def lorenz_small(n: int | None = None, seed_offset: int = 0) -> Problem:
    n = FULL_N["lorenz_small"] if n is None else n
    g = _rng("lorenz_small", seed_offset)
    sigma = g.uniform(8.0, 12.0, n)
    rho = g.uniform(20.0, 36.0, n)
    beta = g.uniform(2.0, 3.0, n)
    eps = g.normal(0.0, np.sqrt(0.01), n)
    u0 = np.stack([1.0 + eps, eps, eps])
    return Problem("lorenz", "tsit5", "f64", n, 3, 3, np.stack([sigma, rho, beta]), u0, 0.0, 1.0,
                   np.array([1.0]), 1e-8, 1e-8, "sumsq", name="lorenz_small")


def lorenz_1m(n: int | None = None, dtype: str = "f64", seed_offset: int = 0) -> Problem:
    n = FULL_N["lorenz_1m"] if n is None else n
    g = _rng("lorenz_1m", seed_offset)
    sigma = g.uniform(8.0, 12.0, n)
    rho = g.uniform(20.0, 36.0, n)
    beta = g.uniform(2.0, 3.0, n)
    eps = g.normal(0.0, np.sqrt(0.01), n)
    u0 = np.stack([1.0 + eps, eps, eps])
    target = g.normal(0.0, 1.0, (10, 3, n))
    prob = Problem("lorenz", "tsit5", "f64", n, 3, 3, np.stack([sigma, rho, beta]), u0, 0.0, 10.0,
                   np.arange(1.0, 11.0), 1e-6, 1e-6, "sumsq", target=target, name="lorenz_1m")
    return prob.as_dtype(dtype)


def robertson(n: int | None = None, seed_offset: int = 0) -> Problem:
    n = FULL_N["robertson"] if n is None else n
    g = _rng("robertson", seed_offset)
    k = np.array([0.04, 3e7, 1e4])[:, None] * np.exp(g.normal(0.0, 0.1, (3, n)))
    u0 = np.zeros((3, n))
    u0[0] = 1.0
    w = g.uniform(0.0, 1.0, (1, 3, n))
    return Problem("robertson", "ros2", "f64", n, 3, 3, k, u0, 0.0, 1e5, np.array([1e5]), 1e-6, 1e-10,
                   "linear", weight=w, name="robertson")


def node64(n: int | None = None, seed_offset: int = 0, dtype: str = "f32") -> Problem:
    n = FULL_N["node64"] if n is None else n
    g = _rng("node64", seed_offset)
    W = g.normal(0.0, np.sqrt(1.0 / 64.0), (64, 64))
    b = g.normal(0.0, np.sqrt(0.1), (64, n))
    u0 = g.normal(0.0, 1.0, (64, n))
    prob = Problem("node64", "tsit5", "f64", n, 64, 64, b, u0, 0.0, 1.0, np.array([1.0]), 1e-5, 1e-5,
                   "sumsq", W=W, name="node64")
    return prob.as_dtype(dtype)


KIN8_RATES = np.array([800.0, 400.0, 2.0, 0.2, 0.05, 0.025, 6.0, 0.004])
KIN8_U0 = np.array([1.0, 0.0, 0.5, 0.0, 0.0, 0.0, 0.3, 0.0])


def kin8(n: int | None = None, seed_offset: int = 0) -> Problem:
    n = FULL_N["kin8"] if n is None else n
    g = _rng("kin8", seed_offset)
    k = KIN8_RATES[:, None] * np.exp(g.normal(0.0, 0.05, (8, n)))
    u0 = np.repeat(KIN8_U0[:, None], n, axis=1)
    return Problem("kin8", "ros3", "f64", n, 8, 8, k, u0, 0.0, 100.0, np.array([100.0]), 1e-7, 1e-7, "sumsq",
                   name="kin8")


def by_name(name: str, n: int | None = None, dtype: str | None = None, seed_offset: int = 0) -> Problem:
    if name == "lorenz_small":
        return lorenz_small(n, seed_offset)
    if name == "lorenz_1m":
        return lorenz_1m(n, dtype or "f64", seed_offset)
    if name == "robertson":
        return robertson(n, seed_offset)
    if name == "node64":
        return node64(n, seed_offset, dtype or "f32")
    if name == "kin8":
        return kin8(n, seed_offset)
    if name == "hires":
        raise NotImplementedError("hires: the HIRES equations and constants are not available here")
    raise KeyError(name)


def scalar_linear(p_values, t1: float = 1.0, method: str = "tsit5") -> Problem:
    """u' = p u, u(0) = 1 per trajectory: the test equation used by the pins."""
    p = np.asarray(p_values, np.float64)[None, :]
    n = p.shape[1]
    return Problem("linear", method, "f64", n, 1, 1, p, np.ones((1, n)), 0.0, t1, np.array([t1]), 1e-8, 1e-8,
                   "linear", weight=np.ones((1, 1, n)), name="linear")
