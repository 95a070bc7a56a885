"""Pins of the oracle's gradient (the tape) by routes that share nothing with it.

* forward-mode dual numbers through the same replay (a second AD route);
* central finite differences with the mesh held FIXED (perturb p / u0 and
  replay the same h; never re-record), with one Richardson level -- GRADSOLVE's
  exactness definition excludes the derivative of the step-size choices
  (evolve.pub review FAQ "Is gradsolve's gradient really exact?");
* brute force on tiny ensembles: the replay in 50-digit decimal arithmetic
  from the exact binary values of the inputs and the tableau, differentiated
  by a 1e-20 central difference (error far below 1e-25);
* invariants: permuting trajectories permutes outputs bitwise, trajectories
  are independent, leading zero steps change nothing bitwise, and the d=64
  shared-weight gradient of an ensemble is the sum of its members'.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest

import oracle
import workloads as W


def _relinf(a, b):
    """Per-trajectory relative error: ||a_i - b_i||_inf / ||b_i||_inf."""
    a = np.vstack(a)
    b = np.vstack(b)
    return np.abs(a - b).max(0) / np.abs(b).max(0)


def _ros3(prob):
    prob.method = "ros3"
    return prob


def _vern7(prob):
    prob.method = "vern7"
    return prob


CASES = {
    "lorenz_small": lambda: W.lorenz_small(48),
    "lorenz_1m": lambda: W.lorenz_1m(24),
    "robertson": lambda: W.robertson(8),
    "robertson_ros3": lambda: _ros3(W.robertson(8)),
    "lorenz_ros3": lambda: _ros3(W.lorenz_small(16)),
    "lorenz_vern7": lambda: _vern7(W.lorenz_small(16)),
}


@pytest.fixture(scope="module")
def recorded():
    out = {}
    for k, f in CASES.items():
        prob = f()
        mesh = oracle.record(prob, W.SMAX[prob.name] * (2 if k.startswith("robertson") else 1)
                             * (32 if k == "lorenz_ros3" else 1))
        assert (mesh.status == 0).all()
        out[k] = (prob, mesh)
    return out


@pytest.mark.parametrize("case", list(CASES))
def test_tape_matches_dual(recorded, case):
    prob, mesh = recorded[case]
    gt = oracle.grad(prob, mesh, "tape")
    gd = oracle.grad(prob, mesh, "dual")
    assert np.array_equal(gt["loss"], gd["loss"])  # same forward arithmetic
    e = _relinf([gt["dp"], gt["du0"]], [gd["dp"], gd["du0"]])
    # the two routes round differently at every step: allow eps per step
    # (Lorenz: ~5e-14 .. 1e-13; Robertson's ~13,000 ROS2 steps: ~3e-12)
    tol = max(1e-13, np.finfo(float).eps * mesh.nsteps.max())
    assert e.max() <= tol, (e.max(), tol)


@pytest.mark.parametrize("case", list(CASES))
def test_fused_tape_matches_dual(recorded, case):
    """The tape with fused adjoint updates (a third plain-precision route,
    which the GPU parity gate uses to gauge what rounding costs on each
    trajectory) computes the same derivative: within eps per step of the
    dual numbers, like the tape, with the same forward values.  Its rounding
    differs from the tape's on the chaotic ensemble."""
    prob, mesh = recorded[case]
    gf = oracle.grad(prob, mesh, "tape_fused")
    gd = oracle.grad(prob, mesh, "dual")
    assert np.array_equal(gf["loss"], gd["loss"])
    e = _relinf([gf["dp"], gf["du0"]], [gd["dp"], gd["du0"]])
    tol = max(1e-13, np.finfo(float).eps * mesh.nsteps.max())
    assert e.max() <= tol, (e.max(), tol)
    if case == "lorenz_1m":
        gt = oracle.grad(prob, mesh, "tape")
        assert not np.array_equal(gf["du0"], gt["du0"])


@pytest.mark.parametrize("case", ["lorenz_small", "robertson", "robertson_ros3", "lorenz_vern7"])
def test_tape_matches_fixed_mesh_fd(recorded, case):
    prob, mesh = recorded[case]
    prob = prob.subset(range(4))
    ns = mesh.nsteps[:4].copy()
    if case.startswith("robertson"):
        # the first 600 steps (t ~ 1e-3, through the stiff transient): the
        # 13,000-step chain's rounding noise would swamp a difference quotient
        ns = np.minimum(ns, 600).astype(np.int32)
    mesh = oracle.Mesh(mesh.h[:4], ns, ns[:, None].copy(), mesh.status[:4], mesh.nreject[:4])
    g = oracle.grad(prob, mesh, "tape")
    base = np.vstack([prob.p, prob.u0])
    # difference steps: relative for the rate constants, absolute for states;
    # Robertson's y2 lives near 1e-5, so its step is 1e-6
    scale = np.ones(base.shape[0])
    if case.startswith("robertson"):
        scale[4] = 1e-2
    fd = np.zeros_like(base)
    for r in range(base.shape[0]):
        for i in range(prob.n):
            x = base[r, i]
            e = 1e-4 * (abs(x) if (case.startswith("robertson") and r < 3) else max(scale[r], abs(x)))

            def Lat(delta):
                pp = base.copy()
                pp[r, i] = x + delta
                q = prob.subset(range(prob.n))
                q.p, q.u0 = pp[: prob.np_], pp[prob.np_:]
                return oracle.replay(q, mesh)[0][i]

            d1 = (Lat(e) - Lat(-e)) / (2 * e)
            d2 = (Lat(e / 2) - Lat(-e / 2)) / e
            fd[r, i] = (4 * d2 - d1) / 3  # Richardson: O(e^4)
    e = _relinf([g["dp"], g["du0"]], [fd[: prob.np_], fd[prob.np_:]])
    # Richardson-extrapolated central differences reach ~1e-9 on Lorenz; on the
    # stiff Robertson chain the loss carries rounding noise that a difference
    # quotient divides by the step, so its floor is ~1e-8..1e-7 (the exact
    # check for ROS2 is the decimal brute force below)
    assert e.max() <= (1e-8 if not case.startswith("robertson") else 1e-7), e


def test_dot_product_node64():
    """<dL/db, db> + <dL/du0, du0> + <dL/dW, dW> = directional derivative (fp64)."""
    prob = W.node64(6, dtype="f64")
    prob = prob.as_dtype("f64")
    mesh = oracle.record(prob, 64)
    g = oracle.grad(prob, mesh, "tape")
    rng = np.random.default_rng(3)
    dpd = rng.normal(size=prob.p.shape)
    dud = rng.normal(size=prob.u0.shape)
    dWd = rng.normal(size=(64, 64))
    lhs = (g["dp"] * dpd).sum() + (g["du0"] * dud).sum() + (g["dW"] * dWd).sum()
    rhs = oracle.dirderiv(prob, mesh, dpd, dud, dWd).sum()
    assert abs(lhs - rhs) <= 1e-12 * max(abs(rhs), np.abs(g["dW"]).sum())


def test_node64_fixed_mesh_fd_on_W():
    prob = W.node64(3, dtype="f64").as_dtype("f64")
    mesh = oracle.record(prob, 64)
    g = oracle.grad(prob, mesh, "tape")
    for (r, c) in [(0, 0), (5, 17), (63, 2)]:
        e = 1e-4

        def Lat(delta):
            q = prob.subset(range(prob.n))
            q.W = prob.W.copy()
            q.W[r, c] += delta
            return oracle.replay(q, mesh)[0].sum()

        d1 = (Lat(e) - Lat(-e)) / (2 * e)
        d2 = (Lat(e / 2) - Lat(-e / 2)) / e
        fd = (4 * d2 - d1) / 3
        assert abs(g["dW"][r, c] - fd) <= 1e-8 * max(1.0, np.abs(g["dW"]).max())


# ---- brute force in 50-digit decimal ------------------------------------------
getcontext().prec = 50


def _dec_tsit5_lorenz(u, p, hs):
    c, A, bt = oracle.tsit5_tableau()
    A = [[Decimal(float(x)) for x in row] for row in A]
    s, r, b = p

    def f(x):
        return [s * (x[1] - x[0]), x[0] * (r - x[2]) - x[1], x[0] * x[1] - b * x[2]]

    for h in hs:
        k = [f(u)]
        for j in range(1, 7):
            U = [u[q] + h * sum(A[j][m] * k[m][q] for m in range(j)) for q in range(3)]
            if j == 6:
                u = U
                break
            k.append(f(U))
    return u


def _dec_ros2_robertson(u, p, hs):
    g = Decimal(oracle.ros2_gamma())
    k1c, k2c, k3c = p

    def f(y):
        r1, r2, r3 = k1c * y[0], k2c * y[1] * y[1], k3c * y[1] * y[2]
        return [r3 - r1, r1 - r3 - r2, r2]

    def J(y):
        return [[-k1c, k3c * y[2], k3c * y[1]],
                [k1c, -k3c * y[2] - 2 * k2c * y[1], -k3c * y[1]],
                [Decimal(0), 2 * k2c * y[1], Decimal(0)]]

    def solve(M, rhs):
        M = [row[:] + [v] for row, v in zip(M, rhs)]
        for k in range(3):
            piv = max(range(k, 3), key=lambda i: abs(M[i][k]))
            M[k], M[piv] = M[piv], M[k]
            for i in range(k + 1, 3):
                l = M[i][k] / M[k][k]
                for j in range(k, 4):
                    M[i][j] -= l * M[k][j]
        x = [Decimal(0)] * 3
        for i in range(2, -1, -1):
            x[i] = (M[i][3] - sum(M[i][j] * x[j] for j in range(i + 1, 3))) / M[i][i]
        return x

    for h in hs:
        Jm = J(u)
        M = [[(1 if i == j else 0) - g * h * Jm[i][j] for j in range(3)] for i in range(3)]
        k1 = solve(M, f(u))
        v = [u[q] + h * k1[q] for q in range(3)]
        fv = f(v)
        k2 = solve(M, [fv[q] - 2 * k1[q] for q in range(3)])
        u = [u[q] + h * (Decimal(3) / 2 * k1[q] + Decimal(1) / 2 * k2[q]) for q in range(3)]
    return u


@pytest.mark.parametrize("case", ["lorenz", "robertson"])
def test_bruteforce_decimal_tiny(case):
    if case == "lorenz":
        prob = W.lorenz_small(3)
        hs_all = [[0.031, 0.017, 0.044, 0.012], [0.02, 0.02, 0.02], [0.05, 0.001, 0.03, 0.04]]
        run = _dec_tsit5_lorenz
        loss = lambda u, i: sum(x * x for x in u)
    else:
        prob = W.robertson(2)
        hs_all = [[1e-6, 3e-6, 1e-5, 4e-5], [2e-6, 1e-5, 1e-4]]
        run = _dec_ros2_robertson
        loss = lambda u, i: sum(Decimal(float(prob.weight[0, q, i])) * u[q] for q in range(3))
    n = len(hs_all)
    prob = prob.subset(range(n))
    S = max(len(x) for x in hs_all)
    h = np.zeros((n, S))
    for i, hs in enumerate(hs_all):
        h[i, : len(hs)] = hs
    ns = np.array([len(x) for x in hs_all], np.int32)
    mesh = oracle.Mesh(h, ns, ns[:, None].copy(), np.zeros(n, np.int32), np.zeros(n, np.int32))
    g = oracle.grad(prob, mesh, "tape", nthreads=1)
    step = Decimal("1e-20")
    for i in range(n):
        hs = [Decimal(float(x)) for x in hs_all[i]]
        x0 = [Decimal(float(v)) for v in np.concatenate([prob.p[:, i], prob.u0[:, i]])]
        ref = []
        for r in range(6):
            xp, xm = list(x0), list(x0)
            xp[r] += step
            xm[r] -= step
            Lp = loss(run(xp[3:], xp[:3], hs), i)
            Lm = loss(run(xm[3:], xm[:3], hs), i)
            ref.append(float((Lp - Lm) / (2 * step)))
        ref = np.array(ref)
        got = np.concatenate([g["dp"][:, i], g["du0"][:, i]])
        assert np.abs(got - ref).max() <= 1e-14 * np.abs(ref).max(), (i, got, ref)
        L = float(loss(run(x0[3:], x0[:3], hs), i))
        assert abs(g["loss"][i] - L) <= 1e-14 * abs(L)


def test_invariants(recorded):
    prob, mesh = recorded["lorenz_1m"]
    g = oracle.grad(prob, mesh, "tape")
    # permutation -> permuted outputs, bitwise
    perm = np.random.default_rng(1).permutation(prob.n)
    gp = oracle.grad(prob.subset(perm), oracle.Mesh(mesh.h[perm], mesh.nsteps[perm], mesh.save_idx[perm],
                                                     mesh.status[perm], mesh.nreject[perm]), "tape")
    for k in ("loss", "dp", "du0"):
        assert np.array_equal(gp[k][..., :] if k == "loss" else gp[k], g[k][perm] if k == "loss" else g[k][:, perm])
    # independence: a subset alone gives the same bits
    sub = [3, 11, 17]
    gs = oracle.grad(prob.subset(sub), oracle.Mesh(mesh.h[sub], mesh.nsteps[sub], mesh.save_idx[sub],
                                                    mesh.status[sub], mesh.nreject[sub]), "tape")
    assert np.array_equal(gs["dp"], g["dp"][:, sub]) and np.array_equal(gs["du0"], g["du0"][:, sub])
    # leading zero-size steps are exact identities for the value and the gradient
    z = 3
    hz = np.concatenate([np.zeros((prob.n, z)), mesh.h], 1)
    gz = oracle.grad(prob, oracle.Mesh(hz, mesh.nsteps + z, mesh.save_idx + z, mesh.status, mesh.nreject), "tape")
    for k in ("loss", "dp", "du0"):
        assert np.array_equal(gz[k], g[k])


def test_node64_shared_gradient_is_member_sum():
    prob = W.node64(4, dtype="f64").as_dtype("f64")
    mesh = oracle.record(prob, 64)
    g = oracle.grad(prob, mesh, "tape", nthreads=1)
    acc = np.zeros((64, 64))
    for i in range(prob.n):
        gi = oracle.grad(prob.subset([i]), oracle.Mesh(mesh.h[[i]], mesh.nsteps[[i]], mesh.save_idx[[i]],
                                                       mesh.status[[i]], mesh.nreject[[i]]), "tape", nthreads=1)
        acc += gi["dW"]
    assert np.abs(acc - g["dW"]).max() <= 1e-13 * np.abs(g["dW"]).max()
