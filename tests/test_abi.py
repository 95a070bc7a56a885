"""The C-ABI library loads and exports every entry point the header declares;
host-side argument validation and workspace sizing (no device work).

The validation tests hand the library placeholder device pointers (address
16) and oversized workspace sizes that only its argument checks stand
between and a launch.  They run in a child process with the GPU hidden
(CUDA_VISIBLE_DEVICES empty), so that a check that regressed would make a
launch fail with a CUDA error instead of touching a real device; each also
checks that the library's launch counter did not move."""
import ctypes
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gradsolve.h")
GPU_HIDDEN = os.environ.get("CUDA_VISIBLE_DEVICES") == ""
hidden_only = pytest.mark.skipif(not GPU_HIDDEN, reason="runs in the GPU-hidden child process "
                                                          "(test_host_checks_with_gpu_hidden)")


@pytest.fixture
def no_launch():
    from discrete_adjoint_b200.gradsolve import _lib
    before = _lib.gs_launch_count()
    yield
    assert _lib.gs_launch_count() == before, "a host-side check reached a kernel launch"


@pytest.mark.skipif(GPU_HIDDEN, reason="this is the child process")
def test_host_checks_with_gpu_hidden():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-m", "pytest", os.path.abspath(__file__), "-q", "-m", "not gpu",
                        "-p", "no:cacheprovider"], env=env, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    passed = re.search(r"(\d+) passed", r.stdout.splitlines()[-1])
    assert passed and int(passed.group(1)) >= 12, r.stdout[-2000:]


def _declared():
    src = open(HEADER).read()
    return re.findall(r"GS_API\s+[\w\s\*]+?\b(gs_\w+)\s*\(", src)


def test_header_declares_entry_points():
    names = set(_declared())
    assert {"gs_workspace_bytes", "gs_count", "gs_record", "gs_solve", "gs_solve_adaptive", "gs_grad", "gs_sens",
            "gs_status_string", "gs_launch_count"} <= names


def test_library_exports_every_declared_symbol():
    import discrete_adjoint_b200 as gs
    lib = ctypes.CDLL(gs.gradsolve.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name


def test_status_strings():
    import discrete_adjoint_b200 as gs
    for code in (0, -1, -2, -3, -4):
        assert gs.gs_status_string(code) not in ("", "unknown status")
    assert gs.gs_status_string(17) == "unknown status"


def _host_problem(n=1000, system=1, method=1, dtype=2, nsave=10, tsave=None):
    from discrete_adjoint_b200.gradsolve import _Problem
    ts = tsave if tsave is not None else [float(k) for k in range(1, nsave + 1)]
    arr = (ctypes.c_double * len(ts))(*ts)
    p = _Problem(system, method, dtype, 3, 3, n, 16, 16, None, 0.0, 10.0, len(ts), arr)
    p._keep = arr
    return p


@hidden_only
def test_workspace_sizes_host_only(no_launch):
    from discrete_adjoint_b200.gradsolve import _Mesh, _lib
    p = _host_problem()
    m = _Mesh(500, 10, None, None, None, None, None, None)
    # one checkpointed state per step and slot, then (Tsit5 on Lorenz) the
    # loss gradient of each save point
    assert _lib.gs_workspace_bytes(ctypes.byref(p), ctypes.byref(m), 1) == (500 * 3 + 10 * 3) * 1000 * 8
    assert _lib.gs_workspace_bytes(ctypes.byref(p), ctypes.byref(m), 0) >= 1000 * 4
    assert _lib.gs_workspace_bytes(ctypes.byref(p), ctypes.byref(m), 7) == 0
    p32 = _host_problem(dtype=1)
    assert _lib.gs_workspace_bytes(ctypes.byref(p32), ctypes.byref(m), 1) == (500 * 3 + 10 * 3) * 1000 * 4


@hidden_only
@pytest.mark.parametrize("bad", ["tsave_order", "tsave_range", "nsave0", "system", "dims", "dtype", "hires"])
def test_invalid_problems_rejected_before_launch(bad, no_launch):
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol
    kw = {}
    if bad == "tsave_order":
        kw["tsave"] = [1.0, 3.0, 2.0]
    if bad == "tsave_range":
        kw["tsave"] = [11.0]
    if bad == "nsave0":
        kw["tsave"] = []
    p = _host_problem(**kw)
    if bad == "system":
        p.system = 9
    if bad == "dims":
        p.d = 4
    if bad == "dtype":
        p.dtype = 3
    if bad == "hires":
        p.system = 3
    tol = _Tol(1e-6, 1e-6, 0.0)
    rc = _lib.gs_count(ctypes.byref(p), ctypes.byref(tol), 100, ctypes.c_void_p(16), None, None)
    assert rc == (-4 if bad == "hires" else -1)
    rc = _lib.gs_solve_adaptive(ctypes.byref(p), ctypes.byref(tol), 100, ctypes.c_void_p(16), None, None, None)
    assert rc == (-4 if bad == "hires" else -1)
    m = _Mesh(100, p.nsave, 16, 16, 16, 16, 16, 16)
    assert _lib.gs_record(ctypes.byref(p), ctypes.byref(tol), ctypes.byref(m), ctypes.c_void_p(16), 1 << 40,
                          None) == (-4 if bad == "hires" else -1)


@hidden_only
def test_bad_tolerance_and_workspace_rejected(no_launch):
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol, _Loss
    p = _host_problem()
    m = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
    assert _lib.gs_count(ctypes.byref(p), ctypes.byref(_Tol(-1.0, 1e-6, 0.0)), 100, ctypes.c_void_p(16), None,
                         None) == -1
    assert _lib.gs_count(ctypes.byref(p), ctypes.byref(_Tol(float("nan"), 1e-6, 0.0)), 100,
                         ctypes.c_void_p(16), None, None) == -1
    # record and grad refuse a workspace that is too small (before any launch)
    assert _lib.gs_record(ctypes.byref(p), ctypes.byref(_Tol(1e-6, 1e-6, 0.0)), ctypes.byref(m),
                          ctypes.c_void_p(16), 8, None) == -3
    ls = _Loss(1, None, None)
    assert _lib.gs_grad(ctypes.byref(p), ctypes.byref(m), ctypes.byref(ls), ctypes.c_void_p(16),
                        ctypes.c_void_p(16), ctypes.c_void_p(16), None, ctypes.c_void_p(16), 8, None) == -3
    # linear loss without weights
    assert _lib.gs_grad(ctypes.byref(p), ctypes.byref(m), ctypes.byref(_Loss(2, None, None)), ctypes.c_void_p(16),
                        ctypes.c_void_p(16), ctypes.c_void_p(16), None, ctypes.c_void_p(16), 1 << 40, None) == -1
    # the adaptive solve needs its output, a capacity and a valid tolerance
    tol = _Tol(1e-6, 1e-6, 0.0)
    assert _lib.gs_solve_adaptive(ctypes.byref(p), ctypes.byref(tol), 100, None, None, None, None) == -1
    assert _lib.gs_solve_adaptive(ctypes.byref(p), ctypes.byref(tol), 0, ctypes.c_void_p(16), None, None,
                                  None) == -1
    assert _lib.gs_solve_adaptive(ctypes.byref(p), ctypes.byref(_Tol(0.0, 0.0, 0.0)), 100, ctypes.c_void_p(16),
                                  None, None, None) == -1
    # forward sensitivities: Tsit5 on Lorenz, ROS2 / ROS3 on both d = 3 systems;
    # the gradient outputs are required
    ls = _Loss(1, None, None)
    assert _lib.gs_sens(ctypes.byref(p), ctypes.byref(m), ctypes.byref(ls), None, ctypes.c_void_p(16),
                        ctypes.c_void_p(16), None, None) == -1
    rob = _host_problem(system=2, method=1)
    assert _lib.gs_sens(ctypes.byref(rob), ctypes.byref(m), ctypes.byref(ls), ctypes.c_void_p(16),
                        ctypes.c_void_p(16), ctypes.c_void_p(16), None, None) == -4
    # mesh nsave must match
    m2 = _Mesh(100, 3, 16, 16, 16, 16, 16, 16)
    assert _lib.gs_solve(ctypes.byref(p), ctypes.byref(m2), ctypes.c_void_p(16), None) == -1


@hidden_only
def test_empty_ensemble_is_a_no_op(no_launch):
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol, _Loss
    p = _host_problem(n=0)
    m = _Mesh(100, 10, None, None, None, None, None, None)
    before = _lib.gs_launch_count()
    assert _lib.gs_count(ctypes.byref(p), ctypes.byref(_Tol(1e-6, 1e-6, 0.0)), 100, None, None, None) == 0
    assert _lib.gs_record(ctypes.byref(p), ctypes.byref(_Tol(1e-6, 1e-6, 0.0)), ctypes.byref(m), None, 0,
                          None) == 0
    assert _lib.gs_grad(ctypes.byref(p), ctypes.byref(m), ctypes.byref(_Loss(1, None, None)), None, None, None,
                        None, None, 0, None) == 0
    assert _lib.gs_solve(ctypes.byref(p), ctypes.byref(m), None, None) == 0
    assert _lib.gs_solve_adaptive(ctypes.byref(p), ctypes.byref(_Tol(1e-6, 1e-6, 0.0)), 100, None, None, None,
                                  None) == 0
    assert _lib.gs_sens(ctypes.byref(p), ctypes.byref(m), ctypes.byref(_Loss(1, None, None)), None, None, None,
                        None, None) == 0
    assert _lib.gs_launch_count() == before


def test_set_option_host_only():
    from discrete_adjoint_b200.gradsolve import _lib
    assert _lib.gs_set_option(1, 1) == 0 and _lib.gs_set_option(1, 0) == 0
    assert _lib.gs_set_option(1, 2) == -1 and _lib.gs_set_option(99, 0) == -1


@hidden_only
def test_ros3_method_validation_host_only(no_launch):
    """ROS3 (method 3) is accepted for the d = 3 systems, dense records and
    sensitivities on dense meshes included; an unknown method is an invalid
    argument.  No call here reaches a launch (the dense paths are checked on
    an empty ensemble)."""
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol, _Loss
    m = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
    ls = _Loss(1, None, None)
    for system in (1, 2):
        p = _host_problem(system=system, method=3)
        assert _lib.gs_workspace_bytes(ctypes.byref(p), ctypes.byref(m), 1) == 100 * 3 * 1000 * 8
        md = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
        md.save_theta = 16
        dense = _Tol(1e-6, 1e-6, 0.0)
        dense.dense = 1
        e = _host_problem(n=0, system=system, method=3)
        assert _lib.gs_count(ctypes.byref(e), ctypes.byref(dense), 100, None, None, None) == 0
        assert _lib.gs_sens(ctypes.byref(e), ctypes.byref(md), ctypes.byref(ls), None, None, None, None, None) == 0
        assert _lib.gs_count(ctypes.byref(e), ctypes.byref(_Tol(1e-6, 1e-6, 0.0)), 100, None, None, None) == 0
    bad = _host_problem(method=5)
    assert _lib.gs_count(ctypes.byref(bad), ctypes.byref(_Tol(1e-6, 1e-6, 0.0)), 100, ctypes.c_void_p(16), None,
                         None) == -1


@hidden_only
def test_vern7_validation_host_only(no_launch):
    """Verner's 7(6) pair (method 4) is accepted for the d = 3 systems with
    landing records; dense records, the d = 8 and d = 64 systems, and a
    gradient or forward sensitivities off Lorenz are not built.  The gradient
    workspace is one checkpointed state per step and slot plus each save
    point's loss gradient.  No call here reaches a launch."""
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol, _Loss
    m = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
    ls = _Loss(1, None, None)
    tol = _Tol(1e-6, 1e-6, 0.0)
    dense = _Tol(1e-6, 1e-6, 0.0)
    dense.dense = 1
    lor = _host_problem(method=4)
    assert _lib.gs_workspace_bytes(ctypes.byref(lor), ctypes.byref(m), 1) == (100 * 3 + 10 * 3) * 1000 * 8
    for system in (1, 2):
        e = _host_problem(n=0, system=system, method=4)
        assert _lib.gs_count(ctypes.byref(e), ctypes.byref(tol), 100, None, None, None) == 0
        assert _lib.gs_count(ctypes.byref(e), ctypes.byref(dense), 100, None, None, None) == -4
        assert _lib.gs_sens(ctypes.byref(e), ctypes.byref(m), ctypes.byref(ls), None, None, None, None,
                            None) == (0 if system == 1 else -4)
        md = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
        md.save_theta = 16
        assert _lib.gs_solve(ctypes.byref(e), ctypes.byref(md), None, None) == -4
    rob = _host_problem(n=0, system=2, method=4)
    assert _lib.gs_grad(ctypes.byref(rob), ctypes.byref(m), ctypes.byref(ls), None, None, None, None, None, 0,
                        None) == -4
    k8 = _host_problem(n=0, system=5, method=4)
    k8.d = k8.np = 8
    assert _lib.gs_count(ctypes.byref(k8), ctypes.byref(tol), 100, None, None, None) == -4


@hidden_only
def test_kin8_validation_host_only(no_launch):
    """kin8 (system 5, d = np = 8) takes ROS2 / ROS3, forward sensitivities
    included (on landing meshes); Tsit5 and dense records are not built for
    it; wrong sizes are invalid.  The gradient workspace is one checkpointed
    8-state per step and slot.  No call here reaches a launch (the accepted
    sensitivities are checked on an empty ensemble)."""
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol, _Loss
    m = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
    ls = _Loss(1, None, None)
    tol = _Tol(1e-7, 1e-7, 0.0)
    for method in (2, 3):
        p = _host_problem(system=5, method=method)
        p.d = p.np = 8
        assert _lib.gs_workspace_bytes(ctypes.byref(p), ctypes.byref(m), 1) == 100 * 8 * 1000 * 8
        md = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
        md.save_theta = 16
        assert _lib.gs_sens(ctypes.byref(p), ctypes.byref(md), ctypes.byref(ls), ctypes.c_void_p(16),
                            ctypes.c_void_p(16), ctypes.c_void_p(16), None, None) == -4
        dense = _Tol(1e-7, 1e-7, 0.0)
        dense.dense = 1
        assert _lib.gs_count(ctypes.byref(p), ctypes.byref(dense), 100, ctypes.c_void_p(16), None, None) == -4
        e = _host_problem(n=0, system=5, method=method)
        e.d = e.np = 8
        assert _lib.gs_count(ctypes.byref(e), ctypes.byref(tol), 100, None, None, None) == 0
        assert _lib.gs_sens(ctypes.byref(e), ctypes.byref(m), ctypes.byref(ls), None, None, None, None, None) == 0
        wrong = _host_problem(system=5, method=method)  # d = np = 3
        assert _lib.gs_count(ctypes.byref(wrong), ctypes.byref(tol), 100, ctypes.c_void_p(16), None, None) == -1
    t5 = _host_problem(system=5, method=1)
    t5.d = t5.np = 8
    assert _lib.gs_count(ctypes.byref(t5), ctypes.byref(tol), 100, ctypes.c_void_p(16), None, None) == -4


@hidden_only
def test_record_inplace_validation_host_only(no_launch):
    """gs_record_inplace refuses before any launch: a missing, small or
    misaligned workspace, the d = 64 system, a dense request without save
    positions, bad tolerances; an empty ensemble is a no-op."""
    from discrete_adjoint_b200.gradsolve import _lib, _Mesh, _Tol
    p = _host_problem()
    m = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
    tol = _Tol(1e-6, 1e-6, 0.0)
    call = lambda prob, mesh, t, ws, nb: _lib.gs_record_inplace(ctypes.byref(prob), ctypes.byref(t),
                                                                ctypes.byref(mesh), ws, nb, None)
    assert call(p, m, tol, None, 8) == -3
    assert call(p, m, tol, ctypes.c_void_p(16), 4) == -3
    assert call(p, m, tol, ctypes.c_void_p(20), 8) == -1
    assert call(p, m, _Tol(-1.0, 1e-6, 0.0), ctypes.c_void_p(16), 8) == -1
    assert call(p, m, _Tol(1e-6, 1e-6, 0.0, 1), ctypes.c_void_p(16), 8) == -1  # dense needs save_theta
    from discrete_adjoint_b200.gradsolve import _Problem
    node = _Problem(4, 1, 1, 64, 64, 1000, 16, 16, 16, 0.0, 10.0, 10, p._keep)
    m64 = _Mesh(100, 10, 16, 16, 16, 16, 16, 16)
    assert call(node, m64, tol, ctypes.c_void_p(16), 8) == -4
    assert call(p, _Mesh(100, 10, 16, None, 16, 16, 16, 16), tol, ctypes.c_void_p(16), 8) == -1  # no order
    assert call(_host_problem(n=0), _Mesh(100, 10, None, None, None, None, None, None), tol, None, 0) == 0
    # the ordered adaptive solve: order and output required, workspace checked
    osv = lambda prob, order, out, ws, nb: _lib.gs_solve_adaptive_ordered(
        ctypes.byref(prob), ctypes.byref(tol), 100, order, out, None, None, ws, nb, None)
    assert osv(p, None, ctypes.c_void_p(16), ctypes.c_void_p(16), 8) == -1
    assert osv(p, ctypes.c_void_p(16), None, ctypes.c_void_p(16), 8) == -1
    assert osv(p, ctypes.c_void_p(16), ctypes.c_void_p(16), None, 8) == -3
    assert osv(p, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 7) == -3
    assert osv(p, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(12), 8) == -1
    assert osv(node, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 8) == -4
    assert osv(_host_problem(n=0), None, None, None, 0) == 0
