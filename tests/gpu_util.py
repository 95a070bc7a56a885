"""Helpers for the GPU tests: move a workloads.Problem to the device, carry an
oracle mesh into the library's slot layout, and read a device mesh back in
trajectory order.  Marshalling only."""
import dataclasses

import numpy as np
import torch

import discrete_adjoint_b200 as gs


def dev():
    return torch.device("cuda:0")


def tens(a, dtype, d=None):
    return torch.tensor(np.ascontiguousarray(a), dtype=dtype, device=d or dev())


def ensemble(prob):
    td = gs.gradsolve.TORCH_DTYPE[prob.dtype]
    return gs.Ensemble(prob.system, prob.method, prob.dtype, tens(prob.p, td), tens(prob.u0, td), prob.t0,
                       prob.t1, [float(x) for x in prob.tsave],
                       None if prob.W is None else tens(prob.W, td))


def loss_args(prob):
    td = gs.gradsolve.TORCH_DTYPE[prob.dtype]
    tgt = None if prob.target is None else tens(prob.target, td)
    w = None if prob.weight is None else tens(prob.weight, td)
    return dict(loss=prob.loss, target=tgt, weight=w)


def mesh_from_oracle(om, dtype, order=None, smax=None):
    """Slot j holds trajectory order[j] (identity by default)."""
    n = om.h.shape[0]
    order = np.arange(n) if order is None else np.asarray(order)
    smax = smax or om.h.shape[1]
    h = np.zeros((smax, n))
    h[: om.h.shape[1]] = om.h[order].T[:smax]
    td = gs.gradsolve.TORCH_DTYPE[dtype]
    i32 = lambda a: tens(np.asarray(a, np.int32), torch.int32)
    theta = None if om.theta is None else tens(om.theta[order].T, td)
    return gs.Mesh(tens(h, td), i32(order), i32(om.nsteps[order]), i32(om.save_idx[order].T),
                   i32(om.status[order]), i32(om.nreject[order]), theta)


def mesh_by_trajectory(mesh):
    """(h [n][smax], nsteps [n], save_idx [n][nsave], status [n], order) in trajectory order."""
    order = mesh.order.cpu().numpy()
    inv = np.empty_like(order)
    inv[order] = np.arange(len(order))
    h = mesh.h.double().cpu().numpy().T[inv]
    return h, mesh.nsteps.cpu().numpy()[inv], mesh.save_idx.cpu().numpy().T[inv], mesh.status.cpu().numpy()[inv], order


def theta_by_trajectory(mesh):
    """save_theta [n][nsave] in trajectory order (a dense record)."""
    order = mesh.order.cpu().numpy()
    inv = np.empty_like(order)
    inv[order] = np.arange(len(order))
    return mesh.save_theta.double().cpu().numpy().T[inv]


def grad_rel_err(out, ref):
    """Per-trajectory ||g - g_ref||_inf / ||g_ref||_inf over (dp, du0)."""
    g = np.vstack([out.dp.double().cpu().numpy(), out.du0.double().cpu().numpy()])
    r = np.vstack([ref["dp"], ref["du0"]])
    return np.abs(g - r).max(0) / np.abs(r).max(0)


def mesh_rel_err(h_gpu, h_orc, ns):
    worst = 0.0
    for i in range(len(ns)):
        a, b = h_gpu[i, : ns[i]], h_orc[i, : ns[i]]
        worst = max(worst, float(np.max(np.abs(a - b) / np.abs(b))) if ns[i] else 0.0)
    return worst


TOL = {"f64": 1e-12, "f32": 1e-4}


def _relinf(g, r):
    return np.abs(g - r).max(0) / np.abs(r).max(0)


# Per-trajectory allowance over the oracle's own plain-precision error.
ROUTE_FACTOR = 4.0


def route_error(prob, om, ref, dual=True):
    """kappa_i: the largest per-trajectory error, against `ref`, of the
    oracle's own plain-precision routes on the same mesh: its tape, the tape
    with fused adjoint updates, and its dual numbers where built.  Each is
    one draw of what rounding in this precision costs on trajectory i (on a
    chaotic trajectory a few amplified roundings dominate, so single draws
    differ by up to ~20x); the largest of three is a steadier gauge."""
    import oracle
    k = None
    for mode in ("tape", "tape_fused") + (("dual",) if dual and prob.system != "node64" else ()):
        g = oracle.grad(prob, om, mode)
        e = _relinf(np.vstack([g["dp"], g["du0"]]), ref)
        k = e if k is None else np.maximum(k, e)
    return k


def parity(out, prob, om, tol=None, c=ROUTE_FACTOR, dual=True):
    """Gradient parity of a GPU result against the oracle on the oracle's mesh.

    Reference: the oracle's tape with a wide reverse sweep (the most accurate
    evaluation of the exact discrete adjoint here).  Error: per trajectory,
    e_i = ||g - g_ref||_inf / ||g_ref||_inf over (dp, du0).  Gate, for every
    trajectory i: e_i <= max(tol, c kappa_i), tol the stated gate (1e-12
    fp64, 1e-4 fp32) and kappa_i the oracle's own plain-precision error on
    that trajectory (route_error).  So the GPU may miss the stated gate only
    on a trajectory where the oracle's own evaluation in the same precision
    misses it too, and then by at most the factor c.  Returns e."""
    import oracle
    tol = tol or TOL[prob.dtype]
    wide = oracle.grad(prob, om, "tape_wide")
    r = np.vstack([wide["dp"], wide["du0"]])
    g = np.vstack([out.dp.double().cpu().numpy(), out.du0.double().cpu().numpy()])
    e = _relinf(g, r)
    over = e > tol
    if over.any():
        kappa = np.zeros_like(e)
        kappa[:] = route_error(prob, om, r, dual)
        bound = np.maximum(tol, c * kappa)
        w = int(np.argmax(e / bound))
        assert (e <= bound).all(), (f"{int((e > bound).sum())} of {len(e)} trajectories over the gate; worst {w}: "
                                    f"error {e[w]:.3e}, oracle routes {kappa[w]:.3e}, bound {bound[w]:.3e}")
    return e


def sens_wide(prob, om, mode="tape_wide"):
    """The sensitivity matrices [nsave][d][np + d][n] from the oracle's tape
    (by default with a wide reverse sweep): one linear loss per (save point,
    component) whose weight selects that entry."""
    K, d, npar = len(prob.tsave), prob.d, prob.np_
    S = np.zeros((K, d, npar + d, prob.n))
    import oracle
    for k in range(K):
        for c in range(d):
            w = np.zeros((K, d, prob.n))
            w[k, c] = 1.0
            q = dataclasses.replace(prob, loss="linear", weight=w, target=None)
            g = oracle.grad(q, om, mode=mode)
            S[k, c, :npar], S[k, c, npar:] = g["dp"], g["du0"]
    return S


def sens_rel(a, ref):
    """Per trajectory: the largest entry error over the largest entry."""
    return np.abs(a - ref).max(axis=(0, 1, 2)) / np.abs(ref).max(axis=(0, 1, 2))


def sens_parity(S, prob, om, tol, c=ROUTE_FACTOR):
    """The gradient criterion applied to the matrices, per trajectory: every
    trajectory within max(tol, c kappa_i), kappa_i the largest error of the
    oracle's own plain-precision routes (dual numbers, the tape, the tape
    with fused updates) on it against the wide reference."""
    import oracle
    ref = sens_wide(prob, om)
    e = sens_rel(S, ref)
    kappa = np.maximum.reduce([sens_rel(oracle.sens(prob, om), ref), sens_rel(sens_wide(prob, om, "tape"), ref),
                               sens_rel(sens_wide(prob, om, "tape_fused"), ref)])
    bound = np.maximum(tol, c * kappa)
    w = int(np.argmax(e / bound))
    assert (e <= bound).all(), (int((e > bound).sum()), w, e[w], kappa[w])
    return e
