"""Pins of the oracle's integrators against facts fixed outside the oracle.

* Tsit5 tableau: the Runge-Kutta order conditions (order 5 for the
  propagating weights, order 4 for the embedded weights b - bt, c = A 1).
* Fixed-step Tsit5 derivative: the gradient printed by the DiffEqGPU
  documentation ("Enzyme reverse mode with EnsembleGPUKernel") for u' = p u,
  20 steps of 0.05 (tests/golden/diffeqgpu_enzyme_tsit5.txt).
* Discrete adjoint on u' = -lambda u: the closed form built from the method's
  stability function R(z) on the mesh (GRADSOLVE's exactness definition: the
  derivative of the fixed-step replay with the mesh held fixed), evaluated in
  exact rational arithmetic.
* ROS2: L-stability (R(inf) = 0 for gamma = 1 + 1/sqrt 2), second order
  (R(z) = 1 + z + z^2/2 + O(z^3)), and the same closed-form adjoint.
* ROS3: the same closed-form adjoint, with R(z) = 1 + z b^T (I - z beta)^{-1} 1
  of the standard Rosenbrock form recovered from the oracle's transformed-form
  coefficients (the coefficient pins themselves are in test_oracle_ros3.py).
* Verner's 7(6) pair: every order condition (all rooted trees up to order 7,
  generated here, in exact rationals of the stored doubles) for b, up to
  order 6 for the embedded weights, which fail at order 7; c = A 1; its step
  on u' = p u equals R(z) = 1 + z b^T (I - z A)^{-1} 1; the same closed-form
  adjoint.
"""
import itertools
import os
from fractions import Fraction as Fr
from math import factorial

import numpy as np
import pytest

import oracle
import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden")
EPS = np.finfo(np.float64).eps


def _tab():
    c, A, bt = oracle.tsit5_tableau()
    b = A[6].copy()                      # propagating weights (FSAL row)
    A6 = np.zeros((7, 7))
    A6[:, :6] = A
    b7 = np.append(b, 0.0)
    return c, A6, b7, bt


def test_tsit5_row_sums():
    c, A, b, bt = _tab()
    assert np.max(np.abs(A.sum(1) - c)) <= 4 * EPS


# Butcher order conditions written as (tree functional, 1/gamma(tree)).
def _conditions(A, c, w, order):
    e = np.ones(len(c))
    conds = [(w @ e, 1.0)]
    if order >= 2:
        conds += [(w @ c, 1 / 2)]
    if order >= 3:
        conds += [(w @ c**2, 1 / 3), (w @ (A @ c), 1 / 6)]
    if order >= 4:
        conds += [(w @ c**3, 1 / 4), (w @ (c * (A @ c)), 1 / 8), (w @ (A @ c**2), 1 / 12),
                  (w @ (A @ (A @ c)), 1 / 24)]
    if order >= 5:
        conds += [(w @ c**4, 1 / 5), (w @ (c**2 * (A @ c)), 1 / 10), (w @ ((A @ c) ** 2), 1 / 20),
                  (w @ (c * (A @ c**2)), 1 / 15), (w @ (c * (A @ (A @ c))), 1 / 30),
                  (w @ (A @ c**3), 1 / 20), (w @ (A @ (c * (A @ c))), 1 / 40),
                  (w @ (A @ (A @ c**2)), 1 / 60), (w @ (A @ (A @ (A @ c))), 1 / 120)]
    return conds


def test_tsit5_order_conditions():
    c, A, b, bt = _tab()
    res5 = [abs(v - t) for v, t in _conditions(A, c, b, 5)]
    assert len(res5) == 17 and max(res5) <= 8 * EPS
    bhat = b - bt
    res4 = [abs(v - t) for v, t in _conditions(A, c, bhat, 4)]
    assert len(res4) == 8 and max(res4) <= 8 * EPS
    # the pair really is 5(4): the embedded weights fail a fifth-order condition
    assert max(abs(v - t) for v, t in _conditions(A, c, bhat, 5)[8:]) > 1e-4


# ---- Verner's 7(6) pair -------------------------------------------------------
def _rooted_trees(order):
    """All rooted trees with ``order`` nodes, each a sorted tuple of its
    subtrees (unlabelled, so each tree appears once)."""
    if order == 1:
        return [()]
    out = set()

    def partitions(n, largest):
        if n == 0:
            yield []
            return
        for k in range(min(n, largest), 0, -1):
            for rest in partitions(n - k, k):
                yield [k] + rest

    for part in partitions(order - 1, order - 1):
        for kids in itertools.product(*[_rooted_trees(k) for k in part]):
            out.add(tuple(sorted(kids)))
    return sorted(out)


def _tree_gamma(t):
    n = 1 + sum(_tree_size(k) for k in t)
    g = n
    for k in t:
        g *= _tree_gamma(k)
    return g


def _tree_size(t):
    return 1 + sum(_tree_size(k) for k in t)


def _elementary_weight(A, t):
    """Phi_i(t) = prod over the subtrees u of (A Phi(u))_i."""
    s = len(A)
    v = [Fr(1)] * s
    for k in t:
        pk = _elementary_weight(A, k)
        Apk = [sum(A[i][j] * pk[j] for j in range(s)) for i in range(s)]
        v = [v[i] * Apk[i] for i in range(s)]
    return v


def _vern7_exact():
    c, A9, b, bh = oracle.vern7_tableau()
    A = [[Fr(float(A9[i, j])) if j < 9 else Fr(0) for j in range(10)] for i in range(10)]
    return [Fr(float(x)) for x in c], A, [Fr(float(x)) for x in b], [Fr(float(x)) for x in bh]


def test_vern7_row_sums_and_tree_count():
    c, A, b, bh = _vern7_exact()
    for i in range(10):
        assert abs(float(sum(A[i]) - c[i])) <= 4 * EPS * sum(abs(float(x)) for x in A[i]), i
    # 1, 1, 2, 4, 9, 20, 48 trees of orders 1..7 (85 conditions in all)
    assert [len(_rooted_trees(k)) for k in range(1, 8)] == [1, 1, 2, 4, 9, 20, 48]


def test_vern7_order_conditions():
    c, A, b, bh = _vern7_exact()
    worst_b7 = worst_bh6 = 0.0
    worst_bh7 = 0.0
    for order in range(1, 8):
        for t in _rooted_trees(order):
            phi = _elementary_weight(A, t)
            want = Fr(1, _tree_gamma(t))
            for w, kind in ((b, "b"), (bh, "bh")):
                got = sum(w[i] * phi[i] for i in range(10))
                mag = float(sum(abs(w[i] * phi[i]) for i in range(10)))
                rel = abs(float(got - want)) / mag
                if kind == "b":
                    worst_b7 = max(worst_b7, rel)
                elif order <= 6:
                    worst_bh6 = max(worst_bh6, rel)
                else:
                    worst_bh7 = max(worst_bh7, rel)
    assert worst_b7 <= 32 * EPS, worst_b7        # seventh order
    assert worst_bh6 <= 64 * EPS, worst_bh6      # sixth-order embedded weights
    assert worst_bh7 > 1e-3, worst_bh7           # ... and not seventh


def _vern7_R_coeffs():
    """R(z) = 1 + sum_k z^(k+1) b^T A^k 1 (A strictly lower triangular)."""
    c, A, b, bh = _vern7_exact()
    v = [Fr(1)] * 10
    co = [Fr(1)]
    for _ in range(10):
        co.append(sum(b[i] * v[i] for i in range(10)))
        v = [sum(A[i][j] * v[j] for j in range(10)) for i in range(10)]
    return co


def test_vern7_stability_function():
    co = _vern7_R_coeffs()
    # seventh order: R agrees with exp to z^7
    assert all(abs(float(co[k] - Fr(1, factorial(k)))) <= 16 * EPS for k in range(8))
    assert abs(float(co[8] - Fr(1, factorial(8)))) > 1e-9
    # one oracle step on u' = p u multiplies u by R(p h)
    for z in [-3.0, -1.0, -0.25, 0.1, 0.5]:
        un, e, ok = oracle.step("linear", "vern7", "f64", np.array([1.0]), np.array([z]), 1.0)
        R = float(_poly(co, Fr(z)))
        terms = float(_poly([abs(x) for x in co], Fr(abs(z))))
        assert abs(un[0] - R) <= 64 * EPS * terms, (z, un[0], R)


def _golden():
    rows = []
    with open(os.path.join(GOLD, "diffeqgpu_enzyme_tsit5.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return np.array(rows)


def _uniform_mesh(n, nsteps, h):
    return oracle.Mesh(np.full((n, nsteps), h), np.full(n, nsteps, np.int32),
                       np.full((n, 1), nsteps, np.int32), np.zeros(n, np.int32), np.zeros(n, np.int32))


@pytest.mark.parametrize("mode", ["tape", "dual"])
def test_worked_example_fixed_step_tsit5(mode):
    g = _golden()
    prob = W.scalar_linear(g[:, 0])
    out = oracle.grad(prob, _uniform_mesh(prob.n, 20, 0.05), mode=mode, nthreads=1)
    rel = np.abs(out["dp"][0] - g[:, 1]) / np.abs(g[:, 1])
    # both codes round differently inside the 20 steps; the printed values
    # differ from exp(p) by 2.6e-14 / 2.1e-13, so 2e-15 pins the DISCRETE derivative
    assert rel.max() <= 2e-15, rel
    assert np.abs(out["dp"][0] - np.exp(g[:, 0])).max() > 1e-14


# ---- closed-form discrete adjoint on u' = p u (p = -lambda) ------------------
def _tsit5_R_coeffs():
    """R(z) = sum_k beta_k z^k: exp's Taylor coefficients up to z^5 (a
    fifth-order method), plus beta_6 = b6 a65 a54 a43 a32 a21 (the only path
    through the strictly lower triangular A), from the exact binary doubles."""
    c, A, b, bt = _tab()
    beta = [Fr(1, factorial(k)) for k in range(6)]
    g6 = Fr(b[5])
    for j in range(5, 0, -1):
        g6 *= Fr(A[j, j - 1])
    return beta + [g6]


def _poly(coeffs, z):
    acc = Fr(0)
    for a in reversed(coeffs):
        acc = acc * z + a
    return acc


def _dpoly(coeffs, z):
    return _poly([k * a for k, a in enumerate(coeffs)][1:], z)


def _ros2_R(z, g):
    num = 1 + (1 - 2 * g) * z + (g * g - 2 * g + Fr(1, 2)) * z * z
    den = (1 - g * z) ** 2
    dnum = (1 - 2 * g) + 2 * (g * g - 2 * g + Fr(1, 2)) * z
    dden = -2 * g * (1 - g * z)
    return num / den, (dnum * den - num * dden) / (den * den)


def _lower_solve(Lm, rhs):
    """Forward substitution with a lower-triangular matrix, exact."""
    x = []
    for i in range(len(rhs)):
        acc = rhs[i] - sum(Lm[i][j] * x[j] for j in range(i))
        x.append(acc / Lm[i][i])
    return x


def _ros3_std():
    """ROS3 in the standard Rosenbrock form (alpha, Gamma, b, bhat), exact
    rationals of the oracle's doubles.  The transformed form's relations
    (Hairer & Wanner, Solving ODEs II, Sec. IV.7): Gamma^{-1} = diag(1/gamma) - C,
    a = alpha Gamma^{-1}, m^T = b^T Gamma^{-1}; the error weights e give the
    embedded solution with weights m - e.  1/gamma is the oracle's rounded
    reciprocal, the value its arithmetic uses."""
    co = oracle.ros3_coeffs()
    ig = Fr(co["inv_gamma"])
    C = [[Fr(0)] * 3, [Fr(co["c21"]), Fr(0), Fr(0)], [Fr(co["c31"]), Fr(co["c32"]), Fr(0)]]
    Ginv = [[(ig if i == j else Fr(0)) - C[i][j] for j in range(3)] for i in range(3)]
    cols = [_lower_solve(Ginv, [Fr(int(i == j)) for i in range(3)]) for j in range(3)]
    G = [[cols[j][i] for j in range(3)] for i in range(3)]
    A = [[Fr(0)] * 3, [Fr(1), Fr(0), Fr(0)], [Fr(1), Fr(0), Fr(0)]]
    alpha = [[sum(A[i][k] * G[k][j] for k in range(3)) for j in range(3)] for i in range(3)]
    m = [Fr(1), Fr(co["m2"]), Fr(co["m3"])]
    e = [Fr(co["e1"]), Fr(co["e2"]), Fr(co["e3"])]
    b = [sum(m[k] * G[k][j] for k in range(3)) for j in range(3)]
    bh = [sum((m[k] - e[k]) * G[k][j] for k in range(3)) for j in range(3)]
    beta = [[alpha[i][j] + G[i][j] for j in range(3)] for i in range(3)]
    return alpha, G, beta, b, bh


_ROS3 = None


def _ros3_R(z):
    """R(z) = 1 + z b^T w and R'(z) = b^T w + z b^T (I - z beta)^{-1} beta w,
    w = (I - z beta)^{-1} 1: the stability function of the standard form."""
    global _ROS3
    if _ROS3 is None:
        _ROS3 = _ros3_std()
    _, _, beta, b, _ = _ROS3
    Mz = [[Fr(int(i == j)) - z * beta[i][j] for j in range(3)] for i in range(3)]
    w = _lower_solve(Mz, [Fr(1)] * 3)
    bw = [sum(beta[i][j] * w[j] for j in range(3)) for i in range(3)]
    y = _lower_solve(Mz, bw)
    bt_w = sum(b[i] * w[i] for i in range(3))
    return 1 + z * bt_w, bt_w + z * sum(b[i] * y[i] for i in range(3))


def _R_any(method, z):
    """(R, R') of Tsit5, Verner 7, ROS2 or ROS3 at z, exact."""
    if method == "tsit5":
        co = _tsit5_R_coeffs()
        return _poly(co, z), _dpoly(co, z)
    if method == "vern7":
        co = _vern7_R_coeffs()
        return _poly(co, z), _dpoly(co, z)
    if method == "ros3":
        return _ros3_R(z)
    return _ros2_R(z, Fr(oracle.ros2_gamma()))


def _closed_form(method, p, hs, u0=Fr(1)):
    """u_N = u0 prod R(z_n), z_n = p h_n; L = u_N^2.
    dL/du0 = 2 u_N prod R(z_n);  dL/dp = 2 u_N^2 sum_n h_n R'(z_n)/R(z_n)."""
    pf = Fr(p)
    R, dR = [], []
    if method == "tsit5":
        co = _tsit5_R_coeffs()
        for h in hs:
            z = pf * Fr(h)
            R.append(_poly(co, z))
            dR.append(_dpoly(co, z))
    else:
        for h in hs:
            r, dr = _R_any(method, pf * Fr(h))
            R.append(r)
            dR.append(dr)
    prod = Fr(1)
    for r in R:
        prod *= r
    uN = u0 * prod
    L = uN * uN
    dL_du0 = 2 * uN * prod
    dL_dp = 2 * L * sum(Fr(h) * dr / r for h, r, dr in zip(hs, R, dR))
    return float(L), float(dL_du0), float(dL_dp)


def _kappa(method, p, hs):
    worst = 1.0
    g = oracle.ros2_gamma()
    co = [float(x) for x in _tsit5_R_coeffs()]
    for h in hs:
        z = p * h
        if method in ("tsit5", "vern7"):
            cm = co if method == "tsit5" else [float(x) for x in _vern7_R_coeffs()]
            terms = sum(abs(a) * abs(z) ** k for k, a in enumerate(cm))
            R = sum(a * z**k for k, a in enumerate(cm))
        elif method == "ros3":
            # |terms| of R = 1 + z b^T w, with |b_i w_i| summed
            if _ROS3 is None:
                _ros3_R(Fr(0))
            beta, b = _ROS3[2], _ROS3[3]
            zf = Fr(z)
            Mz = [[Fr(int(i == j)) - zf * beta[i][j] for j in range(3)] for i in range(3)]
            w = _lower_solve(Mz, [Fr(1)] * 3)
            terms = 1 + abs(z) * sum(abs(float(b[i] * w[i])) for i in range(3))
            R = float(1 + zf * sum(b[i] * w[i] for i in range(3)))
        else:
            d = 1 - g * z
            terms = 1 + 1.5 * abs(z / d) + 0.5 * abs(z * (z * (1 - g) - 1) / d**2)
            R = (1 + (1 - 2 * g) * z + (g * g - 2 * g + 0.5) * z * z) / d**2
        worst = max(worst, terms / abs(R))
    return worst


@pytest.mark.parametrize("method,lams", [("tsit5", [0.5, 3.0, 12.0]), ("ros2", [0.5, 50.0, 1e4]),
                                         ("ros3", [0.5, 50.0, 1e4]), ("vern7", [0.5, 3.0, 12.0])])
@pytest.mark.parametrize("mode", ["tape", "dual"])
def test_closed_form_decay_adjoint(method, lams, mode):
    rng = np.random.default_rng(7)
    N = 25
    hs = rng.uniform(0.005, 0.06, N)
    prob = W.scalar_linear([-l for l in lams], t1=float(hs.sum()), method=method)
    prob.loss = "sumsq"
    prob.weight = None
    n = prob.n
    mesh = oracle.Mesh(np.tile(hs, (n, 1)), np.full(n, N, np.int32), np.full((n, 1), N, np.int32),
                       np.zeros(n, np.int32), np.zeros(n, np.int32))
    out = oracle.grad(prob, mesh, mode=mode, nthreads=1)
    for i, lam in enumerate(lams):
        L, gu, gp = _closed_form(method, -lam, hs)
        # Rounding bound: a step's relative rounding error is about eps times
        # its cancellation factor kappa(z) = (sum of |terms|) / |R(z)| times the
        # size of the method's inner weights (Tsit5: |a_6m| up to ~13, so 32;
        # ROS2: 3/2, 1/2, 2 and gamma, so 8), summed over the N steps.  A
        # wrong digit or a dropped term moves these numbers by 1e-8 or more.
        tol = N * EPS * _kappa(method, -lam, hs) * {"tsit5": 32, "vern7": 128}.get(method, 8)
        assert abs(out["loss"][i] - L) <= tol * abs(L)
        assert abs(out["du0"][0, i] - gu) <= tol * abs(gu)
        assert abs(out["dp"][0, i] - gp) <= tol * abs(gp), (method, lam, out["dp"][0, i], gp)


def test_ros2_stability_function_facts():
    """The ROS2 closed form itself: L-stable (R -> 0 at infinity) and second
    order (Taylor coefficients 1, 1, 1/2), so a slip in the form used above
    would show here."""
    from decimal import Decimal, getcontext
    getcontext().prec = 50
    g = 1 + 1 / Decimal(2).sqrt()
    gf = Fr(str(g))
    r_big, _ = _ros2_R(Fr(-10**30), gf)
    assert abs(float(r_big)) < 1e-25
    eps = Fr(1, 10**6)
    r, _ = _ros2_R(eps, gf)
    assert abs(float((r - 1 - eps - eps * eps / 2) / eps**3)) < 10.0
    # the oracle's gamma is 1 + 1/sqrt(2) to the double's precision
    assert abs(Decimal(oracle.ros2_gamma()) - g) < Decimal(2e-16)


def test_ros2_step_matches_stability_function():
    for lam, h in [(0.7, 0.1), (1e3, 0.05), (3.0, 2.0)]:
        un, _, ok = oracle.step("linear", "ros2", "f64", [1.0], [-lam], h)
        r, _ = _ros2_R(Fr(-lam) * Fr(h), Fr(oracle.ros2_gamma()))
        assert ok and abs(un[0] - float(r)) <= 8 * EPS * max(1.0, abs(float(r)))
