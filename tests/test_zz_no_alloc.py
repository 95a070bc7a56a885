"""gs_grad_static, the gradient entry point for callers that cannot allocate
device memory (its checkpoints live in a library-owned 32 MiB device array),
must give the same results as gs_grad with a caller workspace -- on two calls
in a row with different problems, so a stale array would show.  This file is
collected last, and it passes alone in a fresh process as well."""
import numpy as np
import pytest
import torch

import workloads as W
import discrete_adjoint_b200 as gs
from gpu_util import TOL, dev, ensemble, loss_args

pytestmark = pytest.mark.gpu


def _recorded(prob, smax):
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, smax, len(prob.tsave), prob.dtype, dev())
    gs.gs_record(ens, mesh, prob.rtol, prob.atol)
    nsteps = int(mesh.nsteps.max().item())
    return ens, mesh, nsteps


def _rel(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


def test_static_scratch_matches_workspace_version():
    cases = [W.lorenz_small(), W.lorenz_1m(1000)]
    for call, prob in enumerate(cases):
        ens, mesh, _ = _recorded(prob, 256 if call == 0 else 1024)
        need = gs.gs_workspace_bytes(ens, mesh, gs.gradsolve.OP_GRAD)
        assert need <= gs.gradsolve.STATIC_SCRATCH_BYTES
        ref = gs.gs_grad(ens, mesh, **loss_args(prob))
        got = gs.gs_grad_static(ens, mesh, **loss_args(prob))
        torch.cuda.synchronize()
        for a, b in ((got.loss, ref.loss), (got.dp, ref.dp), (got.du0, ref.du0)):
            assert torch.isfinite(a).all()
            assert _rel(a, b) <= TOL[prob.dtype], (call, _rel(a, b))


def test_static_scratch_rejects_oversize_problems():
    prob = W.lorenz_1m(4096)
    ens = ensemble(prob)
    mesh = gs.new_mesh(prob.n, 1024, len(prob.tsave), prob.dtype, dev())  # 96 MiB of checkpoints
    with pytest.raises(gs.gradsolve.GradsolveError) as e:
        gs.gs_grad_static(ens, mesh, **loss_args(prob))
    assert e.value.code == gs.gradsolve.GS_EWORKSPACE
