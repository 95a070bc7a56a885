"""GPU <-> oracle parity for the adaptive forward-only solve (gs_solve_adaptive):
step counts and statuses equal to the oracle's, saved states within the mesh
bar (1e-10 relative, fp64) or the fp32 bar (1e-4), bitwise equality with the
GPU's own record followed by its replay, failures and ragged sizes, and the
full 2**20-trajectory ensemble checked on a sample."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import dev, ensemble, mesh_by_trajectory

pytestmark = pytest.mark.gpu


def _solve(prob, smax):
    us, ns, st = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, smax)
    torch.cuda.synchronize()
    return us.double().cpu().numpy(), ns.cpu().numpy(), st.cpu().numpy()


def _rel(a, b):
    """Largest error over the largest magnitude, per trajectory (last axis)."""
    return (np.abs(a - b).max(axis=(0, 1)) / np.abs(b).max(axis=(0, 1))).max()


@pytest.mark.parametrize("name,n,smax,bar", [("lorenz_small", 1024, 256, 1e-10), ("lorenz_1m", 4000, 1024, 1e-10),
                                             ("robertson", 700, 20000, 1e-10)])
def test_fp64_matches_oracle(name, n, smax, bar):
    prob = W.by_name(name, n=n)
    ref, rns, rst = oracle.solve_adaptive(prob, smax)
    us, ns, st = _solve(prob, smax)
    assert (rst == 0).all() and np.array_equal(st, rst)
    assert np.array_equal(ns, rns)
    assert _rel(us, ref) <= bar


def test_fp32_matches_oracle():
    prob = W.lorenz_1m(2000, dtype="f32")
    ref, rns, rst = oracle.solve_adaptive(prob, 1024)
    us, ns, st = _solve(prob, 1024)
    assert (st == 0).all() and np.array_equal(ns, rns)
    assert _rel(us, ref) <= 1e-4


@pytest.mark.parametrize("name,dtype,n,smax", [("lorenz_1m", "f64", 3000, 1024), ("lorenz_1m", "f32", 3000, 1024),
                                               ("robertson", "f64", 300, 20000), ("node64", "f32", 300, 64)])
def test_equals_record_then_replay(name, dtype, n, smax):
    """One adaptive iteration, two outputs: the states of the forward-only solve
    are bit for bit those of gs_record followed by gs_solve (for d = 64 with
    either product form: recorder and replay share their stage arithmetic)."""
    for products in ((1, 0) if name == "node64" else (1,)):
        gs.gs_set_option(gs.gradsolve.OPT_NODE64_TENSOR_CORES, products)
        _equals_record_then_replay(name, dtype, n, smax)
    gs.gs_set_option(gs.gradsolve.OPT_NODE64_TENSOR_CORES, 1)


def _equals_record_then_replay(name, dtype, n, smax):
    prob = W.by_name(name, n=n).as_dtype(dtype)
    ens = ensemble(prob)
    us, ns, st = gs.gs_solve_adaptive(ens, prob.rtol, prob.atol, smax)
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), prob.dtype, dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    ur = gs.gs_solve(ens, mesh)
    torch.cuda.synchronize()
    h, mns, si, mst, order = mesh_by_trajectory(mesh)
    assert np.array_equal(ns.cpu().numpy(), mns) and np.array_equal(st.cpu().numpy(), mst)
    assert torch.equal(us, ur)


def test_node64_matches_oracle():
    prob = W.node64(256)
    us, ns, st = _solve(prob, 64)
    assert (st == 0).all()
    # the oracle's replay of the mesh the GPU chose (the fp32 replay bar)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 64, 1, "f32", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, mns, si, mst, order = mesh_by_trajectory(mesh)
    _, ur = oracle.replay(prob, oracle.Mesh(h.astype(np.float64), mns, si, mst, np.zeros(prob.n, np.int32)))
    assert np.abs(us - ur).max() <= 1e-5 * np.abs(ur).max()
    # and the oracle's own adaptive solve: both meet the tolerance (fp32 step
    # decisions differ near err = 1, so the meshes are not identical)
    ref, rns, rst = oracle.solve_adaptive(prob, 64)
    assert (rst == 0).all()
    assert np.abs(us - ref).max() <= 1e-3 * np.abs(ref).max()


def test_failures_and_ragged_sizes():
    prob = W.lorenz_small(129)
    us, ns, st = _solve(prob, 20)  # capacity -> MAXSTEPS everywhere
    assert (st == 1).all() and np.isnan(us).all()
    bad = W.lorenz_small(129)
    bad.p = bad.p.copy()
    bad.p[0, 5] = np.nan
    us, ns, st = _solve(bad, 256)
    ref, rns, rst = oracle.solve_adaptive(bad, 256)
    assert np.array_equal(st, rst) and st[5] == 3 and (np.delete(st, 5) == 0).all()
    assert np.isnan(us[:, :, 5]).all()
    ok = np.delete(np.arange(bad.n), 5)
    assert _rel(us[:, :, ok], ref[:, :, ok]) <= 1e-10
    one = W.lorenz_small(1)
    us, ns, st = _solve(one, 256)
    ref, rns, _ = oracle.solve_adaptive(one, 256)
    assert ns[0] == rns[0] and _rel(us, ref) <= 1e-10


def test_full_size_sampled():
    """2**20 trajectories, fp64, t in [0, 10], ten save points: the oracle checks
    a sample (random + the longest chains) one by one."""
    prob = W.lorenz_1m()
    us, ns, st = gs.gs_solve_adaptive(ensemble(prob), prob.rtol, prob.atol, 2048)
    torch.cuda.synchronize()
    assert (st == 0).all()
    ns_all = ns.cpu().numpy()
    rng = np.random.default_rng(12)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 384, replace=False), np.argsort(ns_all)[-32:]]))
    ref, rns, rst = oracle.solve_adaptive(prob.subset(idx), 2048)
    assert np.array_equal(ns_all[idx], rns)
    got = us[:, :, torch.tensor(idx, device=dev())].cpu().numpy()
    assert _rel(got, ref) <= 1e-10
    assert torch.isfinite(us).all()
    # the benchmark's form: the same solve in a record's slot order, bit for bit
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, int(ns_all.max()), len(prob.tsave), "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    uo, no, so = gs.gs_solve_adaptive_ordered(ens, prob.rtol, prob.atol, 2048, mesh.order)
    torch.cuda.synchronize()
    assert torch.equal(uo, us) and torch.equal(no, ns) and torch.equal(so, st)


@pytest.mark.parametrize("name,method,dtype,dense,n,smax", [
    ("lorenz_1m", None, "f64", False, 4099, 1024), ("lorenz_1m", None, "f64", True, 2051, 1024),
    ("lorenz_1m", None, "f32", False, 2051, 1024), ("robertson", "ros2", "f64", False, 515, 20000),
    ("robertson", "ros3", "f64", True, 515, 4096), ("kin8", "ros3", "f64", False, 333, 8192)])
def test_ordered_equals_unordered(name, method, dtype, dense, n, smax):
    """gs_solve_adaptive_ordered, in a record's slot order and in a random
    order, returns gs_solve_adaptive's states, counts and statuses bit for
    bit (each trajectory's arithmetic does not depend on where it runs)."""
    prob = W.by_name(name, n=n)
    if method:
        prob.method = method
    prob = prob.as_dtype(dtype)
    ens = ensemble(prob)
    ref = [t.cpu().numpy() for t in gs.gs_solve_adaptive(ens, prob.rtol, prob.atol, smax, dense=dense)]
    nst, _ = gs.gs_count(ens, prob.rtol, prob.atol, smax, dense=dense)
    mesh = gs.new_mesh(n, int(nst.max().item()), len(prob.tsave), dtype, dev(), dense=dense)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    rand = torch.tensor(np.random.default_rng(3).permutation(n), dtype=torch.int32, device=dev())
    for order in (mesh.order, rand):
        out = gs.gs_solve_adaptive_ordered(ens, prob.rtol, prob.atol, smax, order, dense=dense)
        torch.cuda.synchronize()
        for a, b in zip(ref, out):
            assert np.array_equal(a, b.cpu().numpy(), equal_nan=True)


def test_ordered_skips_bad_entries():
    """Entries outside [0, n) are skipped: the trajectories no entry names
    keep what their outputs held, the rest are solved."""
    prob = W.lorenz_small(100)
    ens = ensemble(prob)
    ref = [t.cpu().numpy() for t in gs.gs_solve_adaptive(ens, prob.rtol, prob.atol, 256)]
    order = torch.arange(100, dtype=torch.int32, device=dev())
    order[7] = -1
    order[50] = 100
    us = torch.full((len(prob.tsave), 3, 100), 7.0, dtype=torch.float64, device=dev())
    ns = torch.full((100,), -5, dtype=torch.int32, device=dev())
    st = torch.full((100,), -6, dtype=torch.int32, device=dev())
    gs.gs_solve_adaptive_ordered(ens, prob.rtol, prob.atol, 256, order, u_save=us, nsteps=ns, status=st)
    torch.cuda.synchronize()
    us, ns, st = us.cpu().numpy(), ns.cpu().numpy(), st.cpu().numpy()
    skipped = [7, 50]
    keep = np.setdiff1d(np.arange(100), skipped)
    assert (us[..., skipped] == 7.0).all() and (ns[skipped] == -5).all() and (st[skipped] == -6).all()
    assert np.array_equal(us[..., keep], ref[0][..., keep]) and np.array_equal(ns[keep], ref[1][keep])
    assert np.array_equal(st[keep], ref[2][keep])
