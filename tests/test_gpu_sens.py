"""GPU <-> oracle parity for the forward sensitivities (gs_sens) on Lorenz:
the sensitivity matrices d u(t_k) / d (p, u0) against the oracle, the loss
gradient against the adjoint (the same derivative by the other mode), fp64 and
fp32, failures, ragged sizes and the full 2**20-trajectory ensemble on a
sample."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import TOL, dev, ensemble, loss_args, mesh_from_oracle, parity, sens_parity, sens_rel

pytestmark = pytest.mark.gpu


def _run(prob, om, sens=True):
    out, S = gs.gs_sens(ensemble(prob), mesh_from_oracle(om, prob.dtype), sens=sens, **loss_args(prob))
    torch.cuda.synchronize()
    return out, (None if S is None else S.double().cpu().numpy())


def test_small_fp64():
    prob = W.lorenz_small(1024)
    om = oracle.record(prob, 256)
    out, S = _run(prob, om)
    e = sens_rel(S, oracle.sens(prob, om))
    assert e.max() <= 1e-12, e.max()
    sub = prob.subset(np.arange(64))
    sens_parity(S[..., :64], sub, oracle.record(sub, 256), 1e-12)
    loss, _ = oracle.replay(prob, om)
    assert np.abs(out.loss.cpu().numpy() - loss).max() <= 1e-14 * np.abs(loss).max()
    parity(out, prob, om)


@pytest.mark.parametrize("dtype", ["f64", "f32"])
def test_ten_save_points(dtype):
    """t in [0, 10] with ten save points and targets; n not a multiple of 128."""
    prob = W.lorenz_1m(300, dtype=dtype)
    om = oracle.record(prob, 1024)
    out, S = _run(prob, om)
    sens_parity(S, prob, om, TOL[dtype])
    parity(out, prob, om)


def test_gradient_equals_adjoint_on_the_gpu_mesh():
    """Forward and reverse mode give the same derivative of the same replay."""
    prob = W.lorenz_1m(4000)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 1024, 10, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    la = loss_args(prob)
    adj = gs.gs_grad(ens, mesh, **la)
    fwd, _ = gs.gs_sens(ens, mesh, sens=False, **la)
    torch.cuda.synchronize()
    assert torch.equal(fwd.loss, adj.loss)  # the same forward replay, bit for bit
    g_f = torch.cat([fwd.dp, fwd.du0]).cpu().numpy()
    g_a = torch.cat([adj.dp, adj.du0]).cpu().numpy()
    e = np.abs(g_f - g_a).max(0) / np.abs(g_a).max(0)
    assert np.mean(e <= 1e-12) >= 0.99 and e.max() <= 1e-9, (np.mean(e <= 1e-12), e.max())


def test_failures_ragged_and_unsupported():
    prob = W.lorenz_small(129)
    om = oracle.record(prob, 256)
    om.status = om.status.copy()
    om.status[[0, 77]] = 1
    out, S = _run(prob, om)
    assert np.isnan(S[..., [0, 77]]).all() and np.isfinite(np.delete(S, [0, 77], axis=3)).all()
    assert torch.isnan(out.loss[[0, 77]]).all() and torch.isnan(out.dp[:, [0, 77]]).all()
    ok = np.delete(np.arange(prob.n), [0, 77])
    assert sens_rel(np.delete(S, [0, 77], axis=3), oracle.sens(prob, om)[..., ok]).max() <= 1e-12
    out2, none = _run(prob, om, sens=False)
    assert none is None and torch.equal(out2.dp[:, 1:77], out.dp[:, 1:77])
    rob = W.robertson(4)  # Tsit5 forward sensitivities are built for Lorenz only
    rob.method = "tsit5"
    rob.rtol, rob.atol = 1e-3, 1e-6
    with pytest.raises(gs.gradsolve.GradsolveError):
        gs.gs_sens(ensemble(rob), mesh_from_oracle(oracle.record(rob, 20000), "f64"), **loss_args(rob))


def test_full_size_sampled():
    """2**20 trajectories in the launch configuration of the benchmark; the
    oracle checks a sample (random + the longest chains)."""
    prob = W.lorenz_1m()
    ens = ensemble(prob)
    nsteps, _ = gs.gs_count(ens, prob.rtol, prob.atol, 2048)
    smax = int(nsteps.max().item())
    mesh = gs.new_mesh(prob.n, smax, 10, "f64", dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    out, S = gs.gs_sens(ens, mesh, **loss_args(prob))
    torch.cuda.synchronize()
    ns_all = nsteps.cpu().numpy()
    rng = np.random.default_rng(13)
    idx = np.unique(np.concatenate([rng.choice(prob.n, 192, replace=False), np.argsort(ns_all)[-16:]]))
    sub = prob.subset(idx)
    om = oracle.record(sub, 2048)  # equal to the GPU's mesh for these trajectories
    got = S[..., torch.tensor(idx, device=dev())].cpu().numpy()
    sens_parity(got, sub, om, 1e-12)
    assert torch.isfinite(S).all()
