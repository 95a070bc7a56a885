"""CPU oracle for record-and-replay discrete adjoints -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package.  The product (``discrete_adjoint_b200``)
never imports it and shares no code with it.

The oracle is ``oracle.cpp`` compiled with ``-ffp-contract=off`` (so the
compiler never fuses a multiply and an add on its own: every fused
multiply-add is an explicit ``std::fma`` at a site fixed by the floating-point
contract) and loaded through ctypes.  What each entry computes, and the
passage of GRADSOLVE (arXiv 2609.02876) it follows, is documented in
``oracle.cpp``.

Array conventions here: per-trajectory inputs are structure-of-arrays, ``p``
``[np][n]``, ``u0`` ``[d][n]``, ``target``/``weight`` ``[nsave][d][n]``; the
oracle's own mesh is trajectory-major, ``h`` ``[n][smax]``,
``save_idx`` ``[n][nsave]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")

SYSTEMS = {"lorenz": 1, "robertson": 2, "hires": 3, "node64": 4, "linear": 5, "kin8": 6}
METHODS = {"tsit5": 1, "ros2": 2, "ros3": 3, "vern7": 4}
DTYPES = {"f32": 1, "f64": 2}
LOSSES = {"sumsq": 1, "linear": 2}


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to its source (g++, no fused contraction)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-pthread", "-o", _LIB + ".tmp", _SRC]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        i32, i64, f64 = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.or_record.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, dp, f64, f64, i32, dp, f64, f64, f64,
                                i32, dp, ip, ip, ip, ip, i32, dp, i32]
        L.or_grad.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, dp, i32, i32, dp, ip, ip, dp, ip, i32, dp, dp,
                              i32, dp, dp, dp, dp, i32]
        L.or_dirderiv.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, dp, i32, i32, dp, ip, ip, dp, i32, dp, dp,
                                  dp, dp, dp, dp, i32]
        L.or_replay.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, dp, i32, i32, dp, ip, ip, dp, i32, dp, dp,
                                dp, dp, i32]
        L.or_solve_adaptive.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, dp, f64, f64, i32, dp, f64, f64,
                                        f64, i32, i32, dp, ip, ip, i32]
        L.or_sens.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, i32, i32, dp, ip, ip, dp, ip, dp, i32]
        L.or_step_errors.argtypes = [i32, i32, i32, i64, i32, i32, dp, dp, dp, i32, dp, ip, ip, f64, f64, dp, dp,
                                     i32, dp, i32]
        L.or_count_step.argtypes = [i32, i32, i32, i32, dp]
        L.or_step.argtypes = [i32, i32, i32, i32, dp, dp, dp, f64, dp, dp]
        L.or_rhs.argtypes = [i32, i32, dp, dp, dp, dp, dp]
        L.or_tsit5_tableau.argtypes = [dp, dp, dp]
        L.or_tsit5_tableau.restype = None
        L.or_vern7_tableau.argtypes = [dp, dp, dp, dp]
        L.or_vern7_tableau.restype = None
        L.or_tsit5_dense_coeffs.argtypes = [dp]
        L.or_tsit5_dense_coeffs.restype = None
        L.or_tsit5_dense_weights.argtypes = [i32, f64, dp]
        L.or_tsit5_dense_weights.restype = None
        L.or_ros2_gamma.restype = f64
        L.or_ros3_coeffs.argtypes = [dp]
        L.or_ros3_coeffs.restype = None
        L.or_ctrl_pow.argtypes = [i32, i64, dp, dp, dp]
        L.or_ctrl_pow.restype = None
        _lib = L
    return _lib


def _d(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _i(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


@dataclass
class Mesh:
    """The oracle's record: trajectory-major, zero padded."""
    h: np.ndarray         # [n][smax] float64 (fp32 runs hold fp32 values)
    nsteps: np.ndarray    # [n] int32
    save_idx: np.ndarray  # [n][nsave] int32
    status: np.ndarray    # [n] int32
    nreject: np.ndarray   # [n] int32
    theta: np.ndarray | None = None  # [n][nsave] dense-output positions in (0, 1]; None: save points end steps

    @property
    def smax(self) -> int:
        return self.h.shape[1]


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def record(prob, smax: int, h0: float = 0.0, nthreads: int | None = None, dense: bool = False) -> Mesh:
    """Adaptive record of every trajectory of ``prob`` (a ``workloads.Problem``).
    dense: steps do not stop at the save times; each save time is located inside
    its step by theta (the mesh's ``theta``) and read off the step's dense output
    (Tsit5: its own continuous extension; ROS2 / ROS3: the cubic Hermite one)."""
    L = lib()
    n, nsave = prob.n, len(prob.tsave)
    p, u0, W, ts = _f64(prob.p), _f64(prob.u0), _f64(prob.W), _f64(prob.tsave)
    h = np.zeros((n, smax), np.float64)
    nsteps = np.zeros(n, np.int32)
    save_idx = np.zeros((n, max(nsave, 1)), np.int32)
    status = np.zeros(n, np.int32)
    nrej = np.zeros(n, np.int32)
    theta = np.ones((n, max(nsave, 1)), np.float64)
    rc = L.or_record(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[prob.dtype], n, prob.d, prob.np_,
                     _d(p), _d(u0), _d(W), prob.t0, prob.t1, nsave, _d(ts), prob.rtol, prob.atol, h0, smax,
                     _d(h), _i(nsteps), _i(save_idx), _i(status), _i(nrej), int(dense), _d(theta),
                     nthreads or default_threads())
    _check(rc, "record")
    return Mesh(h, nsteps, save_idx[:, :nsave], status, nrej, theta[:, :nsave] if dense else None)


def solve_adaptive(prob, smax: int, h0: float = 0.0, nthreads: int | None = None, dense: bool = False):
    """Adaptive forward-only solve: (u_save [nsave][d][n], nsteps [n], status [n]).
    The recorder's iteration with its accepted states at the save times kept
    (NaN everywhere for a trajectory whose status is not 0)."""
    L = lib()
    n, nsave = prob.n, len(prob.tsave)
    us = np.zeros((nsave, prob.d, n))
    nsteps = np.zeros(n, np.int32)
    status = np.zeros(n, np.int32)
    rc = L.or_solve_adaptive(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[prob.dtype], n, prob.d, prob.np_,
                             _d(_f64(prob.p)), _d(_f64(prob.u0)), _d(_f64(prob.W)), prob.t0, prob.t1, nsave,
                             _d(_f64(prob.tsave)), prob.rtol, prob.atol, h0, smax, int(dense), _d(us), _i(nsteps),
                             _i(status),
                             nthreads or default_threads())
    _check(rc, "solve_adaptive")
    return us, nsteps, status


def _mesh_args(mesh: Mesh):
    h = np.ascontiguousarray(mesh.h, np.float64)
    ns = np.ascontiguousarray(mesh.nsteps, np.int32)
    si = np.ascontiguousarray(mesh.save_idx, np.int32)
    return h, ns, si


def _theta(mesh: Mesh):
    return None if mesh.theta is None else _d(np.ascontiguousarray(mesh.theta, np.float64))


def grad(prob, mesh: Mesh, mode: str = "tape", nthreads: int | None = None):
    """Exact gradient of the fixed-step replay loss.

    mode ``"tape"``: reverse-mode AD (tape).  mode ``"dual"``: forward mode,
    one dual-number pass per input (p and u0; not node64).  mode
    ``"tape_wide"``: the tape with its adjoints accumulated in a wider type
    (long double for fp64, double for fp32).  mode ``"tape_fused"``: the tape
    with every adjoint update as one fused multiply-add (plain precision,
    rounded differently from ``"tape"``).
    Returns dict(loss [n], dp [np][n], du0 [d][n], dW [64,64] or None).
    """
    L = lib()
    n, d, npar = prob.n, prob.d, prob.np_
    h, ns, si = _mesh_args(mesh)
    st = np.ascontiguousarray(mesh.status, np.int32)
    loss = np.zeros(n)
    dp = np.zeros((npar, n))
    du0 = np.zeros((d, n))
    dW = np.zeros((64, 64)) if prob.system == "node64" else None
    rc = L.or_grad(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[prob.dtype], n, d, npar, _d(_f64(prob.p)),
                   _d(_f64(prob.u0)), _d(_f64(prob.W)), mesh.smax, si.shape[1], _d(h), _i(ns), _i(si),
                   _theta(mesh), _i(st), LOSSES[prob.loss], _d(_f64(prob.target)), _d(_f64(prob.weight)), {"tape": 0, "dual": 1, "tape_wide": 2, "tape_fused": 3}[mode],
                   _d(loss), _d(dp), _d(du0), _d(dW), nthreads or default_threads())
    _check(rc, "grad")
    return {"loss": loss, "dp": dp, "du0": du0, "dW": dW}


def dirderiv(prob, mesh: Mesh, dir_p=None, dir_u0=None, dir_W=None, nthreads: int | None = None):
    """Forward-mode directional derivative of each trajectory's loss, [n]."""
    L = lib()
    h, ns, si = _mesh_args(mesh)
    out = np.zeros(prob.n)
    rc = L.or_dirderiv(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[prob.dtype], prob.n, prob.d, prob.np_,
                       _d(_f64(prob.p)), _d(_f64(prob.u0)), _d(_f64(prob.W)), mesh.smax, si.shape[1], _d(h),
                       _i(ns), _i(si), _theta(mesh), LOSSES[prob.loss], _d(_f64(prob.target)),
                       _d(_f64(prob.weight)), _d(_f64(dir_p)), _d(_f64(dir_u0)), _d(_f64(dir_W)), _d(out), nthreads or default_threads())
    _check(rc, "dirderiv")
    return out


def sens(prob, mesh: Mesh, nthreads: int | None = None):
    """Forward sensitivities of the fixed-step replay by dual numbers:
    [nsave][d][np + d][n], column j = d u(t_k) / d (p, u0)_j; NaN rows for
    trajectories whose mesh status is not 0."""
    L = lib()
    h, ns, si = _mesh_args(mesh)
    st = np.ascontiguousarray(mesh.status, np.int32)
    out = np.zeros((si.shape[1], prob.d, prob.np_ + prob.d, prob.n))
    rc = L.or_sens(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[prob.dtype], prob.n, prob.d, prob.np_,
                   _d(_f64(prob.p)), _d(_f64(prob.u0)), mesh.smax, si.shape[1], _d(h), _i(ns), _i(si),
                   _theta(mesh), _i(st), _d(out), nthreads or default_threads())
    _check(rc, "sens")
    return out


def replay(prob, mesh: Mesh, nthreads: int | None = None):
    """Plain replay: (loss [n], u_save [nsave][d][n])."""
    L = lib()
    h, ns, si = _mesh_args(mesh)
    loss = np.zeros(prob.n)
    us = np.zeros((si.shape[1], prob.d, prob.n))
    rc = L.or_replay(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[prob.dtype], prob.n, prob.d, prob.np_,
                     _d(_f64(prob.p)), _d(_f64(prob.u0)), _d(_f64(prob.W)), mesh.smax, si.shape[1], _d(h),
                     _i(ns), _i(si), _theta(mesh), LOSSES[prob.loss], _d(_f64(prob.target)),
                     _d(_f64(prob.weight)), _d(loss), _d(us), nthreads or default_threads())
    _check(rc, "replay")
    return loss, us


def step_errors(prob, mesh: Mesh, dtype: str | None = None, nperturb: int = 0, nthreads: int | None = None):
    """The recorder's view of a given mesh (in `dtype`, default the problem's):
    (err [n][smax], fac [n][smax]) -- each step's scaled error on the replay
    of that mesh and the PI factor accepting it gives (no cap after a
    rejection).  Zeros past nsteps and on trajectories with status != 0.
    nperturb > 0 adds draws [nperturb][n][smax]: the factors again with each
    step's start state perturbed at the precision's epsilon (one draw of
    rounding per evaluation)."""
    L = lib()
    h, ns, _ = _mesh_args(mesh)
    st = np.ascontiguousarray(mesh.status, np.int32)
    err = np.zeros((prob.n, mesh.smax))
    fac = np.zeros((prob.n, mesh.smax))
    draws = np.zeros((nperturb, prob.n, mesh.smax)) if nperturb else None
    rc = L.or_step_errors(SYSTEMS[prob.system], METHODS[prob.method], DTYPES[dtype or prob.dtype], prob.n, prob.d,
                          prob.np_, _d(_f64(prob.p)), _d(_f64(prob.u0)), _d(_f64(prob.W)), mesh.smax, _d(h), _i(ns),
                          _i(st), prob.rtol, prob.atol, _d(err), _d(fac), nperturb, _d(draws),
                          nthreads or default_threads())
    _check(rc, "step_errors")
    return (err, fac, draws) if nperturb else (err, fac)


def count_step(system: str, method: str, d: int, npar: int) -> dict:
    """Arithmetic operations of one fixed replay step (no error estimate)."""
    out = np.zeros(6)
    lib().or_count_step(SYSTEMS[system], METHODS[method], d, npar, _d(out))
    return dict(zip(["add", "mul", "fma", "div", "sqrt", "tanh"], out.astype(int).tolist()))


def step(system: str, method: str, dtype: str, u, p, h: float, W=None):
    """One step of the method: (u_new, error estimate, ok)."""
    u = _f64(u)
    pp = np.zeros(64)
    if p is not None:
        pp[: len(p)] = p
    un = np.zeros_like(u)
    er = np.zeros_like(u)
    rc = lib().or_step(SYSTEMS[system], METHODS[method], DTYPES[dtype], len(u), _d(u), _d(pp), _d(_f64(W)),
                       h, _d(un), _d(er))
    return un, er, rc == 0


def rhs(system: str, u, p, W=None):
    """(f(u), analytic Jacobian or zeros) at one point, float64."""
    u = _f64(u)
    d = len(u)
    f = np.zeros(d)
    J = np.zeros((d, d)) if d <= 8 else None
    lib().or_rhs(SYSTEMS[system], d, _d(u), _d(_f64(p)), _d(_f64(W)), _d(f), _d(J))
    return f, J


def tsit5_tableau():
    c = np.zeros(7)
    A = np.zeros((7, 6))
    bt = np.zeros(7)
    lib().or_tsit5_tableau(_d(c), _d(A), _d(bt))
    return c, A, bt


def vern7_tableau():
    """Verner's 7(6) pair as the oracle holds it: c[10], A[10][9], b[10], bhat[10]."""
    c, A, b, bh = np.zeros(10), np.zeros((10, 9)), np.zeros(10), np.zeros(10)
    lib().or_vern7_tableau(_d(c), _d(A), _d(b), _d(bh))
    return c, A, b, bh


def tsit5_dense_coeffs():
    """r[7][4] of Tsit5's continuous extension: b_i(theta) = sum_m r[i, m-1] theta^m."""
    r = np.zeros((7, 4))
    lib().or_tsit5_dense_coeffs(_d(r))
    return r


def tsit5_dense_weights(theta: float, dtype: str = "f64"):
    """b_1(theta) .. b_7(theta) as the oracle's dense output forms them."""
    bw = np.zeros(7)
    lib().or_tsit5_dense_weights(1 if dtype == "f32" else 2, float(theta), _d(bw))
    return bw


def ros2_gamma() -> float:
    return float(lib().or_ros2_gamma())


def ros3_coeffs() -> dict:
    """The oracle's ROS3 coefficients: gamma, inv_gamma, c21, c31, c32, m2, m3,
    e1, e2, e3 (m1 = 1, a21 = a31 = 1, a32 = 0)."""
    v = np.zeros(10)
    lib().or_ros3_coeffs(_d(v))
    keys = ["gamma", "inv_gamma", "c21", "c31", "c32", "m2", "m3", "e1", "e2", "e3"]
    return dict(zip(keys, (float(x) for x in v)))


def ctrl_pow(x, y, dtype: str = "f64"):
    """The step-size controller's power function x**y, element-wise."""
    x = np.ascontiguousarray(x, np.float64).ravel()
    y = np.broadcast_to(np.asarray(y, np.float64), x.shape).copy()
    out = np.zeros_like(x)
    lib().or_ctrl_pow(DTYPES[dtype], len(x), _d(x), _d(y), _d(out))
    return out
