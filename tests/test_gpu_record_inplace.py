"""GPU parity of gs_record_inplace, the re-record that keeps the slot order an
earlier record set and writes every slot's steps straight into the mesh: the
same mesh as gs_record bit for bit, the oracle's record per trajectory under
any slot order, zero padding kept when step counts shrink, and malformed
order entries marked instead of read."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import dev, ensemble, mesh_by_trajectory

pytestmark = pytest.mark.gpu

# (workload, method override, dtype, dense, n): ragged n so the last group of
# 32 slots is partial
CASES = [("lorenz_small", None, "f64", False, 1000), ("lorenz_1m", None, "f64", False, 4099),
         ("lorenz_1m", None, "f64", True, 2051), ("lorenz_1m", None, "f32", False, 2051),
         ("robertson", "ros2", "f64", False, 515), ("robertson", "ros3", "f64", True, 1027),
         ("robertson", "ros3", "f32", False, 515), ("kin8", "ros3", "f64", False, 333), ("kin8", "ros2", "f64", False, 65),
         ("lorenz_small", None, "f64", False, 1), ("lorenz_small", None, "f64", False, 33)]


def _problem(name, method, dtype, n):
    prob = W.by_name(name, n=n)
    if method:
        prob.method = method
    return prob.as_dtype(dtype)


def _arrays(mesh):
    ts = [mesh.h, mesh.order, mesh.nsteps, mesh.save_idx, mesh.status, mesh.nreject]
    if mesh.save_theta is not None:
        ts.append(mesh.save_theta)
    return [t.cpu().numpy().copy() for t in ts]


def _clone(mesh):
    return gs.Mesh(*[None if t is None else t.clone() for t in (mesh.h, mesh.order, mesh.nsteps, mesh.save_idx,
                                                                mesh.status, mesh.nreject, mesh.save_theta)])


def _sized_mesh(prob, ens, dense):
    cap = 20000 if prob.name == "kin8" else 4 * W.SMAX[prob.name]
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, cap, dense=dense)
    return gs.new_mesh(prob.n, int(nsteps.max().item()), len(prob.tsave), prob.dtype, dev(), dense=dense)


@pytest.mark.parametrize("name,method,dtype,dense,n", CASES)
def test_inplace_equals_record(name, method, dtype, dense, n):
    """After gs_record, gs_record_inplace on the same ensemble rewrites every
    mesh array with the same bits (twice in a row, too)."""
    prob = _problem(name, method, dtype, n)
    ens = ensemble(prob)
    mesh = _sized_mesh(prob, ens, dense)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    ref = _arrays(mesh)
    assert (ref[4] == 0).all()
    again = _clone(mesh)
    for _ in range(2):
        gs.gs_record_inplace(ens, again, prob.rtol, prob.atol)
        torch.cuda.synchronize()
        for a, b in zip(ref, _arrays(again)):
            assert np.array_equal(a, b)


@pytest.mark.parametrize("method", ["tsit5", "ros3"])
def test_inplace_any_order_matches_oracle(method):
    """Under a random slot order (never sorted), each trajectory's steps,
    count, save indices, status and rejections equal the oracle's fp64 record
    bit for bit."""
    prob = _problem("lorenz_small" if method == "tsit5" else "robertson", None if method == "tsit5" else method,
                    "f64", 777)
    om = oracle.record(prob, 4 * W.SMAX[prob.name])
    ens = ensemble(prob)
    smax = int(om.nsteps.max())
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), "f64", dev())
    mesh.order.copy_(torch.tensor(np.random.default_rng(5).permutation(prob.n), dtype=torch.int32))
    gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, ns, si, st, _ = mesh_by_trajectory(mesh)
    assert np.array_equal(ns, om.nsteps) and np.array_equal(st, om.status)
    assert np.array_equal(si, om.save_idx)
    assert np.array_equal(h, om.h[:, :smax])
    nrej = mesh.nreject.cpu().numpy()
    order = mesh.order.cpu().numpy()
    assert np.array_equal(nrej, om.nreject[order])


def test_inplace_shrinking_counts_keep_zero_padding():
    """A tight-tolerance record, then an in-place re-record at a looser
    tolerance: counts shrink, the rows past them are zero again, and every
    trajectory equals a fresh gs_record at the looser tolerance."""
    prob = _problem("lorenz_1m", None, "f64", 1500)
    ens = ensemble(prob)
    tight = gs.gs_count(ens, 1e-9, 1e-9, 8192)[0]
    mesh = gs.new_mesh(prob.n, int(tight.max().item()), len(prob.tsave), "f64", dev())
    gs.gs_record(ens, mesh, 1e-9, 1e-9)
    before = mesh.nsteps.clone()
    gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    assert (mesh.nsteps < before).all()
    hs = mesh.h.cpu().numpy()
    ns = mesh.nsteps.cpu().numpy()
    assert all((hs[ns[j]:, j] == 0).all() and (hs[: ns[j], j] > 0).all() for j in range(prob.n))
    fresh = gs.new_mesh(prob.n, mesh.smax, len(prob.tsave), "f64", dev())
    gs.gs_record(ens, fresh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    a, b = mesh_by_trajectory(mesh), mesh_by_trajectory(fresh)
    for x, y in zip(a[:4], b[:4]):
        assert np.array_equal(x, y)


def test_inplace_bad_order_entries():
    """Order entries outside [0, n) give their slots GS_TRAJ_BADORDER, no steps,
    zeroed rows and save indices; every other slot is recorded as before."""
    prob = _problem("lorenz_small", None, "f64", 200)
    ens = ensemble(prob)
    mesh = _sized_mesh(prob, ens, False)
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    ref = _arrays(mesh)
    bad = [5, 17, 199]
    mesh.order[5] = -1
    mesh.order[17] = prob.n + 3
    mesh.order[199] = 2 ** 31 - 1
    gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    h, order, ns, si, st, nr = _arrays(mesh)
    keep = np.setdiff1d(np.arange(prob.n), bad)
    assert (st[bad] == gs.gradsolve.TRAJ_BADORDER).all() and (ns[bad] == 0).all() and (nr[bad] == 0).all()
    assert (h[:, bad] == 0).all() and (si[:, bad] == 0).all()
    assert np.array_equal(h[:, keep], ref[0][:, keep]) and np.array_equal(ns[keep], ref[2][keep])
    assert np.array_equal(si[:, keep], ref[3][:, keep]) and (st[keep] == 0).all()


def test_inplace_refusals():
    """The d = 64 system has no in-place recorder; a missing or small
    workspace is refused before any launch."""
    prob = W.node64(64)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 64, 1, "f32", dev())
    with pytest.raises(gs.gradsolve.GradsolveError) as e:
        gs.gs_record_inplace(ens, mesh, prob.rtol, prob.atol)
    assert e.value.code == gs.gradsolve.GS_EUNSUPPORTED
    p3 = _problem("lorenz_small", None, "f64", 64)
    e3 = ensemble(p3)
    m3 = gs.new_mesh(p3.n, 64, len(p3.tsave), "f64", dev())
    with pytest.raises(gs.gradsolve.GradsolveError) as e:
        gs.gs_record_inplace(e3, m3, p3.rtol, p3.atol, ws=torch.empty(4, dtype=torch.uint8, device=dev()))
    assert e.value.code == gs.gradsolve.GS_EWORKSPACE


def test_inplace_capacity_failures_match_record():
    """With a capacity below the longest chains, the trajectories that run
    out end with GS_TRAJ_MAXSTEPS and a truncated mesh, the same bits as
    gs_record's (and nothing is written past the capacity)."""
    prob = _problem("lorenz_1m", None, "f64", 1000)
    ens = ensemble(prob)
    ns, _ = gs.gs_count(ens, prob.rtol, prob.atol, 4096)
    cap = int(np.median(ns.cpu().numpy()))
    mesh = gs.new_mesh(prob.n, cap, len(prob.tsave), "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    ref = _arrays(mesh)
    st = ref[4]
    assert (st == gs.gradsolve.TRAJ_MAXSTEPS).sum() > 100 and (st == 0).sum() > 100
    again = _clone(mesh)
    gs.gs_record_inplace(ens, again, prob.rtol, prob.atol)
    torch.cuda.synchronize()
    for a, b in zip(ref, _arrays(again)):
        assert np.array_equal(a, b)
