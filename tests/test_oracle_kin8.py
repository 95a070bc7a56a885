"""Pins of the oracle's d = 8 system kin8 and of its Rosenbrock steps at d = 8.

kin8 is an 8-species stiff mass-action network defined by this library (not a
published test problem): species A1..A8, rate constants k1..k8 for
    A1 -> A2, A2 -> A1, A2 + A3 -> A4, A4 -> A3 + A5,
    A5 -> A6, A6 -> A5, A6 + A7 -> A8, A8 -> A7 + A1.
Its pins, each from a fact outside the oracle's hand-written formulas:

* the right-hand side is the mass-action law of that reaction list,
  f = sum_r (products_r - reactants_r) k_r prod_s u_s^(reactant order), evaluated
  here generically from the list;
* the analytic Jacobian matches central differences of the right-hand side;
* one ROS2 / ROS3 step (8 x 8 LU with partial pivoting) equals the methods'
  stage equations solved with LAPACK (numpy.linalg.solve);
* the three linear invariants u1+u2+u4+u5+u6+u8, u3+u4, u7+u8 (left null
  vectors of the stoichiometric matrix) are conserved by every Rosenbrock
  stage, so recorded solutions keep them to rounding;
* the adaptive ROS3 solution at a tight tolerance agrees with scipy's Radau;
* the gradient: tape = dual numbers, and central differences with the mesh
  held fixed.
"""
import numpy as np
import pytest
from scipy.integrate import solve_ivp

import oracle
import workloads as W

REACTIONS = [  # (reactants, products) with stoichiometric coefficients
    ({0: 1}, {1: 1}),
    ({1: 1}, {0: 1}),
    ({1: 1, 2: 1}, {3: 1}),
    ({3: 1}, {2: 1, 4: 1}),
    ({4: 1}, {5: 1}),
    ({5: 1}, {4: 1}),
    ({5: 1, 6: 1}, {7: 1}),
    ({7: 1}, {6: 1, 0: 1}),
]
INVARIANTS = np.array([[1, 1, 0, 1, 1, 1, 0, 1], [0, 0, 1, 1, 0, 0, 0, 0], [0, 0, 0, 0, 0, 0, 1, 1]], float)


def _stoich():
    N = np.zeros((8, len(REACTIONS)))
    for r, (re, pr) in enumerate(REACTIONS):
        for s, a in re.items():
            N[s, r] -= a
        for s, a in pr.items():
            N[s, r] += a
    return N


def mass_action(u, k):
    rates = np.array([k[r] * np.prod([u[s] ** a for s, a in re.items()]) for r, (re, _) in enumerate(REACTIONS)])
    return _stoich() @ rates


def mass_action_jac(u, k):
    N = _stoich()
    dr = np.zeros((len(REACTIONS), 8))
    for r, (re, _) in enumerate(REACTIONS):
        for s, a in re.items():
            other = np.prod([u[q] ** b for q, b in re.items() if q != s])
            dr[r, s] = k[r] * a * u[s] ** (a - 1) * other
    return N @ dr


def test_invariants_are_left_null_vectors():
    assert np.abs(INVARIANTS @ _stoich()).max() == 0


def test_rhs_is_mass_action():
    rng = np.random.default_rng(8)
    for _ in range(20):
        u = rng.uniform(0.0, 1.0, 8)
        k = W.KIN8_RATES * np.exp(rng.normal(0, 0.3, 8))
        f, J = oracle.rhs("kin8", u, k)
        ref = mass_action(u, k)
        assert np.abs(f - ref).max() <= 8 * np.finfo(float).eps * np.abs(ref).max() * 4
        assert np.abs(J - mass_action_jac(u, k)).max() <= 4 * np.finfo(float).eps * np.abs(J).max()


def test_jacobian_matches_differences():
    rng = np.random.default_rng(9)
    u = rng.uniform(0.05, 1.0, 8)
    k = W.KIN8_RATES.copy()
    _, J = oracle.rhs("kin8", u, k)
    for j in range(8):
        e = 1e-6 * max(abs(u[j]), 1e-3)
        fp, _ = oracle.rhs("kin8", u + e * np.eye(8)[j], k)
        fm, _ = oracle.rhs("kin8", u - e * np.eye(8)[j], k)
        assert np.abs((fp - fm) / (2 * e) - J[:, j]).max() <= 1e-7 * np.abs(J).max()


def _ros_step_lapack(method, u, k, h):
    f = lambda x: mass_action(x, k)
    J = mass_action_jac(u, k)
    if method == "ros2":
        g = oracle.ros2_gamma()
        M = np.eye(8) - g * h * J
        k1 = np.linalg.solve(M, f(u))
        v = u + h * k1
        k2 = np.linalg.solve(M, f(v) - 2 * k1)
        return u + h * (1.5 * k1 + 0.5 * k2), 0.5 * h * (k1 + k2)
    c = oracle.ros3_coeffs()
    M = np.eye(8) / c["gamma"] - h * J
    k1 = np.linalg.solve(M, f(u))
    v = u + h * k1
    fv = f(v)
    k2 = np.linalg.solve(M, fv + c["c21"] * k1)
    k3 = np.linalg.solve(M, fv + c["c31"] * k1 + c["c32"] * k2)
    return u + h * (k1 + c["m2"] * k2 + c["m3"] * k3), h * (c["e1"] * k1 + c["e2"] * k2 + c["e3"] * k3)


@pytest.mark.parametrize("method", ["ros2", "ros3"])
@pytest.mark.parametrize("h", [1e-4, 0.05, 3.0])
def test_rosenbrock_step_matches_lapack(method, h):
    rng = np.random.default_rng(10)
    for _ in range(5):
        u = rng.uniform(0.0, 1.0, 8)
        k = W.KIN8_RATES * np.exp(rng.normal(0, 0.3, 8))
        un, err, ok = oracle.step("kin8", method, "f64", u, k, h)
        ref_un, ref_err = _ros_step_lapack(method, u, k, h)
        assert ok
        # cond(M) ~ 1 + gamma h |lambda_max| (<= ~1e4 here) times eps
        assert np.abs(un - ref_un).max() <= 1e-12 * max(1.0, np.abs(ref_un).max())
        assert np.abs(err - ref_err).max() <= 1e-11 * max(np.abs(ref_err).max(), 1e-300)


@pytest.mark.parametrize("method", ["ros2", "ros3"])
def test_recorded_solution_keeps_invariants(method):
    prob = W.kin8(6)
    prob.method = method
    prob.tsave = np.array([1.0, 10.0, 100.0])
    mesh = oracle.record(prob, 40000)
    assert (mesh.status == 0).all()
    _, us = oracle.replay(prob, mesh)
    c0 = INVARIANTS @ prob.u0
    for k in range(len(prob.tsave)):
        drift = np.abs(INVARIANTS @ us[k] - c0).max()
        assert drift <= 1e-13 * np.sqrt(mesh.nsteps.max()), (k, drift)


def test_tight_tolerance_solution_matches_radau():
    prob = W.kin8(2)
    prob.tsave = np.array([1.0, 30.0, 100.0])
    prob.rtol = prob.atol = 1e-11
    mesh = oracle.record(prob, 200000)
    assert (mesh.status == 0).all()
    _, us = oracle.replay(prob, mesh)
    for i in range(prob.n):
        k = prob.p[:, i]
        ref = solve_ivp(lambda t, y: mass_action(y, k), (0.0, 100.0), prob.u0[:, i], method="Radau",
                        t_eval=prob.tsave, rtol=1e-12, atol=1e-14, jac=lambda t, y: mass_action_jac(y, k))
        assert ref.success
        assert np.abs(us[:, :, i] - ref.y.T).max() <= 1e-8


def test_fixed_step_convergence_orders():
    """ROS2 and ROS3 on kin8 with equal fixed steps over t in [0, 0.002], inside
    the fast pair's transient (h |lambda_fast| <= 0.08, the asymptotic range):
    global error ratios give the orders 2 and 3."""
    prob = W.kin8(1)
    T = 0.002

    def solve(method, N):
        prob.method = method
        m = oracle.Mesh(np.full((1, N), T / N), np.array([N], np.int32), np.array([[N]], np.int32),
                        np.zeros(1, np.int32), np.zeros(1, np.int32))
        return oracle.replay(prob, m)[1][0, :, 0]

    for method, order in (("ros2", 2), ("ros3", 3)):
        ref = solve(method, 8192)
        e1 = np.abs(solve(method, 32) - ref).max()
        e2 = np.abs(solve(method, 64) - ref).max()
        assert abs(np.log2(e1 / e2) - order) < 0.3, (method, np.log2(e1 / e2))


@pytest.mark.parametrize("method", ["ros2", "ros3"])
def test_gradient_tape_matches_dual(method):
    prob = W.kin8(4)
    prob.method = method
    mesh = oracle.record(prob, 40000)
    gt = oracle.grad(prob, mesh, "tape")
    gd = oracle.grad(prob, mesh, "dual")
    assert np.array_equal(gt["loss"], gd["loss"])
    a, b = np.vstack([gt["dp"], gt["du0"]]), np.vstack([gd["dp"], gd["du0"]])
    e = np.abs(a - b).max(0) / np.abs(b).max(0)
    assert e.max() <= max(1e-13, np.finfo(float).eps * mesh.nsteps.max()), e.max()


def test_gradient_matches_fixed_mesh_differences():
    prob = W.kin8(2)
    mesh = oracle.record(prob, 40000)
    g = oracle.grad(prob, mesh, "tape")
    base = np.vstack([prob.p, prob.u0])
    fd = np.zeros_like(base)
    for r in range(base.shape[0]):
        for i in range(prob.n):
            x = base[r, i]
            e = 1e-4 * (abs(x) if r < 8 else 1.0)

            def Lat(delta):
                q = prob.subset(range(prob.n))
                pp = base.copy()
                pp[r, i] = x + delta
                q.p, q.u0 = pp[:8], pp[8:]
                return oracle.replay(q, mesh)[0][i]

            d1 = (Lat(e) - Lat(-e)) / (2 * e)
            d2 = (Lat(e / 2) - Lat(-e / 2)) / e
            fd[r, i] = (4 * d2 - d1) / 3
    a, b = np.vstack([g["dp"], g["du0"]]), fd
    e = np.abs(a - b).max(0) / np.abs(b).max(0)
    assert e.max() <= 1e-8, e


# ---- brute force in 50-digit decimal ------------------------------------------
def _dec_kin8_replay(method, u, p, hs):
    """The ROS2 / ROS3 replay of kin8 in 50-digit decimal arithmetic, written
    from the methods' stage equations with the coefficients as the exact
    binary values the oracle uses; linear systems by Gaussian elimination."""
    from decimal import Decimal as D

    def f(y):
        return [D(x) for x in mass_action_dec(y, p)]

    def J(y):
        return mass_action_jac_dec(y, p)

    def solve(M, rhs):
        A = [row[:] + [v] for row, v in zip(M, rhs)]
        for k in range(8):
            piv = max(range(k, 8), key=lambda i: abs(A[i][k]))
            A[k], A[piv] = A[piv], A[k]
            for i in range(k + 1, 8):
                l = A[i][k] / A[k][k]
                for j in range(k, 9):
                    A[i][j] -= l * A[k][j]
        x = [D(0)] * 8
        for i in range(7, -1, -1):
            x[i] = (A[i][8] - sum(A[i][j] * x[j] for j in range(i + 1, 8))) / A[i][i]
        return x

    for h in hs:
        Jm = J(u)
        if method == "ros2":
            g = D(oracle.ros2_gamma())
            M = [[(D(1) if i == j else D(0)) - g * h * Jm[i][j] for j in range(8)] for i in range(8)]
            k1 = solve(M, f(u))
            v = [u[q] + h * k1[q] for q in range(8)]
            fv = f(v)
            k2 = solve(M, [fv[q] - 2 * k1[q] for q in range(8)])
            u = [u[q] + h * (D(3) / 2 * k1[q] + D(1) / 2 * k2[q]) for q in range(8)]
        else:
            c = {k: D(v) for k, v in oracle.ros3_coeffs().items()}
            M = [[(c["inv_gamma"] if i == j else D(0)) - h * Jm[i][j] for j in range(8)] for i in range(8)]
            k1 = solve(M, f(u))
            v = [u[q] + h * k1[q] for q in range(8)]
            fv = f(v)
            k2 = solve(M, [fv[q] + c["c21"] * k1[q] for q in range(8)])
            k3 = solve(M, [fv[q] + c["c31"] * k1[q] + c["c32"] * k2[q] for q in range(8)])
            u = [u[q] + h * (k1[q] + c["m2"] * k2[q] + c["m3"] * k3[q]) for q in range(8)]
    return u


def mass_action_dec(u, k):
    """mass_action in Decimal arithmetic (u, k lists of Decimal)."""
    N = _stoich()
    rates = []
    for r, (re, _) in enumerate(REACTIONS):
        v = k[r]
        for s, a in re.items():
            for _ in range(a):
                v = v * u[s]
        rates.append(v)
    return [sum(int(N[s, r]) * rates[r] for r in range(len(REACTIONS))) for s in range(8)]


def mass_action_jac_dec(u, k):
    N = _stoich()
    from decimal import Decimal as D
    dr = [[D(0)] * 8 for _ in REACTIONS]
    for r, (re, _) in enumerate(REACTIONS):
        for s, a in re.items():
            other = k[r]
            for q, b in re.items():
                if q != s:
                    for _ in range(b):
                        other = other * u[q]
            dr[r][s] = a * other * (u[s] ** (a - 1) if a > 1 else D(1))
    return [[sum(int(N[i, r]) * dr[r][j] for r in range(len(REACTIONS))) for j in range(8)] for i in range(8)]


@pytest.mark.parametrize("method", ["ros2", "ros3"])
def test_bruteforce_decimal_tiny(method):
    """Two trajectories of 3-4 steps up to h = 0.5 (h |lambda_fast| ~ 600, the
    stiff regime): the oracle's tape gradient and loss against the replay in
    50-digit decimal differentiated by 1e-20 central differences."""
    from decimal import Decimal as D, getcontext
    getcontext().prec = 50
    prob = W.kin8(2)
    prob.method = method
    hs_all = [[0.01, 0.1, 0.5, 0.25], [0.002, 0.3, 0.05]]
    S = max(len(x) for x in hs_all)
    h = np.zeros((2, S))
    for i, hs in enumerate(hs_all):
        h[i, : len(hs)] = hs
    ns = np.array([len(x) for x in hs_all], np.int32)
    mesh = oracle.Mesh(h, ns, ns[:, None].copy(), np.zeros(2, np.int32), np.zeros(2, np.int32))
    g = oracle.grad(prob, mesh, "tape", nthreads=1)
    step = D("1e-20")
    loss = lambda u: sum(x * x for x in u)
    for i in range(2):
        hs = [D(float(x)) for x in hs_all[i]]
        x0 = [D(float(v)) for v in np.concatenate([prob.p[:, i], prob.u0[:, i]])]
        ref = []
        for r in range(16):
            xp, xm = list(x0), list(x0)
            xp[r] += step
            xm[r] -= step
            Lp = loss(_dec_kin8_replay(method, xp[8:], xp[:8], hs))
            Lm = loss(_dec_kin8_replay(method, xm[8:], xm[:8], hs))
            ref.append(float((Lp - Lm) / (2 * step)))
        ref = np.array(ref)
        got = np.concatenate([g["dp"][:, i], g["du0"][:, i]])
        assert np.abs(got - ref).max() <= 1e-14 * np.abs(ref).max(), (i, np.abs(got - ref).max())
        L = float(loss(_dec_kin8_replay(method, x0[8:], x0[:8], hs)))
        assert abs(g["loss"][i] - L) <= 1e-14 * abs(L)
