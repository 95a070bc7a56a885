"""ctypes binding of libgradsolve (include/gradsolve.h).

Argument marshalling only: every function below turns torch tensors into the
C structs and pointers of the ABI and calls the library on the caller's CUDA
stream.  All work runs in the library's kernels; there is no fallback path:
if the shared library is missing this module raises at import.

Record-and-replay discrete adjoints (GRADSOLVE, arXiv 2609.02876): gs_record
stores each trajectory's accepted steps once; gs_grad returns the exact
derivative of the fixed-step replay of that mesh (evolve.pub review,
"Strengths: precisely scoped exactness claim"); gs_solve is the forward-only
replay.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgradsolve.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libgradsolve.so not built ({LIB_PATH}); run `python discrete_adjoint_b200/build.py` "
                      "(or __graft_entry__.build()) first -- there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

# ---- constants (mirroring include/gradsolve.h) -------------------------------
GS_OK, GS_EINVAL, GS_ECUDA, GS_EWORKSPACE, GS_EUNSUPPORTED = 0, -1, -2, -3, -4
TRAJ_OK, TRAJ_MAXSTEPS, TRAJ_DTMIN, TRAJ_NONFINITE, TRAJ_SINGULAR, TRAJ_BADORDER = 0, 1, 2, 3, 4, 5
SYSTEMS = {"lorenz": 1, "robertson": 2, "hires": 3, "node64": 4, "kin8": 5}
METHODS = {"tsit5": 1, "ros2": 2, "ros3": 3, "vern7": 4}
DTYPES = {"f32": 1, "f64": 2}
LOSSES = {"sumsq": 1, "linear": 2}
OP_RECORD, OP_GRAD = 0, 1
RECORD_INPLACE_WS = 8
MAX_SAVE = 64
TORCH_DTYPE = {"f32": torch.float32, "f64": torch.float64}


class _Problem(ctypes.Structure):
    _fields_ = [("system", ctypes.c_int32), ("method", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("d", ctypes.c_int32), ("np", ctypes.c_int32), ("n", ctypes.c_int64),
                ("p", ctypes.c_void_p), ("u0", ctypes.c_void_p), ("shared", ctypes.c_void_p),
                ("t0", ctypes.c_double), ("t1", ctypes.c_double), ("nsave", ctypes.c_int32),
                ("tsave", ctypes.POINTER(ctypes.c_double))]


class _Tol(ctypes.Structure):
    _fields_ = [("rtol", ctypes.c_double), ("atol", ctypes.c_double), ("h0", ctypes.c_double),
                ("dense", ctypes.c_int32)]


class _Mesh(ctypes.Structure):
    _fields_ = [("smax", ctypes.c_int32), ("nsave", ctypes.c_int32), ("h", ctypes.c_void_p),
                ("order", ctypes.c_void_p), ("nsteps", ctypes.c_void_p), ("save_idx", ctypes.c_void_p),
                ("status", ctypes.c_void_p), ("nreject", ctypes.c_void_p), ("save_theta", ctypes.c_void_p)]


class _Loss(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("target", ctypes.c_void_p), ("weight", ctypes.c_void_p)]


_P = ctypes.POINTER
_lib.gs_workspace_bytes.argtypes = [_P(_Problem), _P(_Mesh), ctypes.c_int32]
_lib.gs_workspace_bytes.restype = ctypes.c_size_t
_lib.gs_count.argtypes = [_P(_Problem), _P(_Tol), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.gs_count.restype = ctypes.c_int32
_lib.gs_record.argtypes = [_P(_Problem), _P(_Tol), _P(_Mesh), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
_lib.gs_record.restype = ctypes.c_int32
_lib.gs_record_inplace.argtypes = [_P(_Problem), _P(_Tol), _P(_Mesh), ctypes.c_void_p, ctypes.c_size_t,
                                   ctypes.c_void_p]
_lib.gs_record_inplace.restype = ctypes.c_int32
_lib.gs_solve.argtypes = [_P(_Problem), _P(_Mesh), ctypes.c_void_p, ctypes.c_void_p]
_lib.gs_solve_adaptive.argtypes = [_P(_Problem), _P(_Tol), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p]
_lib.gs_solve_adaptive.restype = ctypes.c_int32
_lib.gs_solve_adaptive_ordered.argtypes = [_P(_Problem), _P(_Tol), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p]
_lib.gs_solve_adaptive_ordered.restype = ctypes.c_int32
_lib.gs_set_option.argtypes = [ctypes.c_int32, ctypes.c_int32]
_lib.gs_set_option.restype = ctypes.c_int32
_lib.gs_sens.argtypes = [_P(_Problem), _P(_Mesh), _P(_Loss)] + [ctypes.c_void_p] * 5
_lib.gs_sens.restype = ctypes.c_int32
_lib.gs_solve.restype = ctypes.c_int32
_lib.gs_grad.argtypes = [_P(_Problem), _P(_Mesh), _P(_Loss), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]
_lib.gs_grad.restype = ctypes.c_int32
_lib.gs_grad_static.argtypes = [_P(_Problem), _P(_Mesh), _P(_Loss), ctypes.c_void_p, ctypes.c_void_p,
                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.gs_grad_static.restype = ctypes.c_int32
STATIC_SCRATCH_BYTES = 32 << 20
_lib.gs_status_string.argtypes = [ctypes.c_int32]
_lib.gs_status_string.restype = ctypes.c_char_p
_lib.gs_launch_count.argtypes = []
_lib.gs_launch_count.restype = ctypes.c_int64


class GradsolveError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {gs_status_string(code)} ({code})")
        self.code = code


def gs_status_string(code: int) -> str:
    return _lib.gs_status_string(code).decode()


def gs_launch_count() -> int:
    return int(_lib.gs_launch_count())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


@dataclass
class Ensemble:
    """An ensemble on the device: p [np][n], u0 [d][n] (and W [64][64] for
    node64), all of the arithmetic dtype, plus its time span and save times."""
    system: str
    method: str
    dtype: str
    p: torch.Tensor
    u0: torch.Tensor
    t0: float
    t1: float
    tsave: list
    shared: torch.Tensor | None = None

    @property
    def n(self) -> int:
        return self.u0.shape[1]

    @property
    def d(self) -> int:
        return self.u0.shape[0]

    @property
    def np_(self) -> int:
        return self.p.shape[0]

    def _struct(self):
        td = TORCH_DTYPE[self.dtype]
        for name, t in (("p", self.p), ("u0", self.u0), ("shared", self.shared)):
            if t is None:
                continue
            if t.dtype != td or not t.is_contiguous() or not t.is_cuda:
                raise ValueError(f"Ensemble.{name} must be a contiguous CUDA {td} tensor")
        ts = (ctypes.c_double * len(self.tsave))(*[float(x) for x in self.tsave])
        s = _Problem(SYSTEMS[self.system], METHODS[self.method], DTYPES[self.dtype], self.d, self.np_, self.n,
                     self.p.data_ptr(), self.u0.data_ptr(), None if self.shared is None else self.shared.data_ptr(),
                     float(self.t0), float(self.t1), len(self.tsave), ts)
        s._keep = ts
        return s


@dataclass
class Mesh:
    """A record on the device, indexed by slot (order[slot] = trajectory)."""
    h: torch.Tensor         # [smax][n] dtype
    order: torch.Tensor     # [n] int32
    nsteps: torch.Tensor    # [n] int32
    save_idx: torch.Tensor  # [nsave][n] int32
    status: torch.Tensor    # [n] int32
    nreject: torch.Tensor   # [n] int32
    save_theta: torch.Tensor | None = None  # [nsave][n] dtype: dense record (position inside the step)

    @property
    def smax(self) -> int:
        return self.h.shape[0]

    @property
    def nsave(self) -> int:
        return self.save_idx.shape[0]

    def _struct(self):
        return _Mesh(self.smax, self.nsave, self.h.data_ptr(), self.order.data_ptr(), self.nsteps.data_ptr(),
                     self.save_idx.data_ptr(), self.status.data_ptr(), self.nreject.data_ptr(),
                     None if self.save_theta is None else self.save_theta.data_ptr())


def new_mesh(n: int, smax: int, nsave: int, dtype: str, device="cuda", dense: bool = False) -> Mesh:
    """Allocate (caller-side, via torch) an empty mesh of capacity smax; dense
    adds the save-point positions a dense record writes."""
    i32 = dict(dtype=torch.int32, device=device)
    td = TORCH_DTYPE[dtype]
    return Mesh(torch.zeros((smax, n), dtype=td, device=device), torch.zeros(n, **i32),
                torch.zeros(n, **i32), torch.zeros((nsave, n), **i32), torch.zeros(n, **i32), torch.zeros(n, **i32),
                torch.ones((nsave, n), dtype=td, device=device) if dense else None)


def gs_workspace_bytes(ens: Ensemble, mesh: Mesh | None, op: int, smax: int | None = None) -> int:
    ps = ens._struct()
    if mesh is not None:
        ms = mesh._struct()
    else:
        ms = _Mesh(smax, len(ens.tsave), None, None, None, None, None, None, None)
    return int(_lib.gs_workspace_bytes(ctypes.byref(ps), ctypes.byref(ms), op))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A caller-owned workspace buffer (torch allocation, 256-byte aligned)."""
    return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)


def _check(rc: int, what: str):
    if rc != GS_OK:
        raise GradsolveError(rc, what)


def gs_count(ens: Ensemble, rtol: float, atol: float, smax: int, h0: float = 0.0, nsteps=None, status=None,
             stream=None, dense: bool = False):
    """Step counts and statuses per TRAJECTORY (sizing pass)."""
    dev = ens.u0.device
    if nsteps is None:
        nsteps = torch.empty(ens.n, dtype=torch.int32, device=dev)
    if status is None:
        status = torch.empty(ens.n, dtype=torch.int32, device=dev)
    ps, tol = ens._struct(), _Tol(rtol, atol, h0, int(dense))
    _check(_lib.gs_count(ctypes.byref(ps), ctypes.byref(tol), smax, _ptr(nsteps), _ptr(status), _stream(stream)),
           "gs_count")
    return nsteps, status


def gs_solve_adaptive(ens: Ensemble, rtol: float, atol: float, smax: int, h0: float = 0.0, u_save=None,
                      nsteps=None, status=None, stream=None, dense: bool = False):
    """Adaptive forward-only solve: (u_save [nsave][d][n], nsteps [n], status [n]),
    all by trajectory; no mesh is kept."""
    dev = ens.u0.device
    if u_save is None:
        u_save = torch.empty((len(ens.tsave), ens.d, ens.n), dtype=TORCH_DTYPE[ens.dtype], device=dev)
    if nsteps is None:
        nsteps = torch.empty(ens.n, dtype=torch.int32, device=dev)
    if status is None:
        status = torch.empty(ens.n, dtype=torch.int32, device=dev)
    ps, tol = ens._struct(), _Tol(rtol, atol, h0, int(dense))
    _check(_lib.gs_solve_adaptive(ctypes.byref(ps), ctypes.byref(tol), smax, _ptr(u_save), _ptr(nsteps),
                                  _ptr(status), _stream(stream)), "gs_solve_adaptive")
    return u_save, nsteps, status


def gs_solve_adaptive_ordered(ens: Ensemble, rtol: float, atol: float, smax: int, order, h0: float = 0.0,
                              u_save=None, nsteps=None, status=None, ws=None, stream=None, dense: bool = False):
    """gs_solve_adaptive with trajectories run in groups of 32 consecutive
    entries of order (device int32 permutation, e.g. an earlier record's
    mesh.order); outputs by trajectory."""
    dev = ens.u0.device
    if u_save is None:
        u_save = torch.empty((len(ens.tsave), ens.d, ens.n), dtype=TORCH_DTYPE[ens.dtype], device=dev)
    if nsteps is None:
        nsteps = torch.empty(ens.n, dtype=torch.int32, device=dev)
    if status is None:
        status = torch.empty(ens.n, dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(RECORD_INPLACE_WS, dev)
    ps, tol = ens._struct(), _Tol(rtol, atol, h0, int(dense))
    _check(_lib.gs_solve_adaptive_ordered(ctypes.byref(ps), ctypes.byref(tol), smax, _ptr(order), _ptr(u_save),
                                          _ptr(nsteps), _ptr(status), _ptr(ws), ws.numel(), _stream(stream)),
           "gs_solve_adaptive_ordered")
    return u_save, nsteps, status


def gs_record(ens: Ensemble, mesh: Mesh, rtol: float, atol: float, h0: float = 0.0, ws=None, stream=None,
              dense: bool | None = None):
    """Adaptive record into mesh; dense (default: whether the mesh carries
    save_theta) records steps that do not stop at the save times."""
    dense = mesh.save_theta is not None if dense is None else dense
    ps, ms, tol = ens._struct(), mesh._struct(), _Tol(rtol, atol, h0, int(dense))
    need = int(_lib.gs_workspace_bytes(ctypes.byref(ps), ctypes.byref(ms), OP_RECORD))
    if ws is None:
        ws = workspace(need, ens.u0.device)
    _check(_lib.gs_record(ctypes.byref(ps), ctypes.byref(tol), ctypes.byref(ms), _ptr(ws), ws.numel(),
                          _stream(stream)), "gs_record")
    return mesh


def gs_record_inplace(ens: Ensemble, mesh: Mesh, rtol: float, atol: float, h0: float = 0.0, ws=None, stream=None,
                      dense: bool | None = None):
    """Re-record into mesh keeping its slot order (set by an earlier record)."""
    dense = mesh.save_theta is not None if dense is None else dense
    ps, ms, tol = ens._struct(), mesh._struct(), _Tol(rtol, atol, h0, int(dense))
    if ws is None:
        ws = workspace(RECORD_INPLACE_WS, ens.u0.device)
    _check(_lib.gs_record_inplace(ctypes.byref(ps), ctypes.byref(tol), ctypes.byref(ms), _ptr(ws), ws.numel(),
                                  _stream(stream)), "gs_record_inplace")
    return mesh


def gs_solve(ens: Ensemble, mesh: Mesh, u_save=None, stream=None):
    if u_save is None:
        u_save = torch.empty((len(ens.tsave), ens.d, ens.n), dtype=TORCH_DTYPE[ens.dtype], device=ens.u0.device)
    ps, ms = ens._struct(), mesh._struct()
    _check(_lib.gs_solve(ctypes.byref(ps), ctypes.byref(ms), _ptr(u_save), _stream(stream)), "gs_solve")
    return u_save


@dataclass
class GradOut:
    loss: torch.Tensor
    dp: torch.Tensor
    du0: torch.Tensor
    dshared: torch.Tensor | None


def new_grad_out(ens: Ensemble) -> GradOut:
    td, dev = TORCH_DTYPE[ens.dtype], ens.u0.device
    return GradOut(torch.empty(ens.n, dtype=td, device=dev), torch.empty((ens.np_, ens.n), dtype=td, device=dev),
                   torch.empty((ens.d, ens.n), dtype=td, device=dev),
                   torch.empty((64, 64), dtype=td, device=dev) if ens.system == "node64" else None)


def gs_grad(ens: Ensemble, mesh: Mesh, loss: str = "sumsq", target=None, weight=None, out: GradOut | None = None,
            ws=None, stream=None) -> GradOut:
    """Loss of the fixed-step replay and its exact discrete adjoint, per trajectory."""
    if out is None:
        out = new_grad_out(ens)
    ps, ms = ens._struct(), mesh._struct()
    ls = _Loss(LOSSES[loss], None if target is None else target.data_ptr(),
               None if weight is None else weight.data_ptr())
    need = int(_lib.gs_workspace_bytes(ctypes.byref(ps), ctypes.byref(ms), OP_GRAD))
    if ws is None:
        ws = workspace(need, ens.u0.device)
    _check(_lib.gs_grad(ctypes.byref(ps), ctypes.byref(ms), ctypes.byref(ls), _ptr(out.loss), _ptr(out.dp),
                        _ptr(out.du0), _ptr(out.dshared), _ptr(ws), ws.numel(), _stream(stream)), "gs_grad")
    return out


OPT_NODE64_TENSOR_CORES = 1


def gs_set_option(option: int, value: int) -> None:
    """Process-wide option (OPT_NODE64_TENSOR_CORES: 1 = the d = 64 products on
    the tensor cores, the default; 0 = SIMT, the recorder's arithmetic)."""
    _check(_lib.gs_set_option(option, value), "gs_set_option")


def gs_sens(ens: Ensemble, mesh: Mesh, loss: str = "sumsq", target=None, weight=None, out: GradOut | None = None,
            sens=True, stream=None):
    """Forward sensitivities of the fixed-step replay: (GradOut with the loss and
    its gradient by forward mode, sens [nsave][d][np + d][n] or None).  Pass
    sens=False to skip the matrices, or a tensor to write them into."""
    if out is None:
        out = new_grad_out(ens)
    if sens is True:
        sens = torch.empty((len(ens.tsave), ens.d, ens.np_ + ens.d, ens.n), dtype=TORCH_DTYPE[ens.dtype],
                           device=ens.u0.device)
    elif sens is False:
        sens = None
    ps, ms = ens._struct(), mesh._struct()
    ls = _Loss(LOSSES[loss], None if target is None else target.data_ptr(),
               None if weight is None else weight.data_ptr())
    _check(_lib.gs_sens(ctypes.byref(ps), ctypes.byref(ms), ctypes.byref(ls), _ptr(out.loss), _ptr(out.dp),
                        _ptr(out.du0), _ptr(sens), _stream(stream)), "gs_sens")
    return out, sens


def gs_grad_static(ens: Ensemble, mesh: Mesh, loss: str = "sumsq", target=None, weight=None,
                   out: GradOut | None = None, stream=None) -> GradOut:
    """gs_grad for callers that cannot allocate device memory: the checkpoints
    go to the library's own 32 MiB device array (problems that need more are
    rejected; calls that overlap on the GPU race)."""
    if out is None:
        out = new_grad_out(ens)
    ps, ms = ens._struct(), mesh._struct()
    ls = _Loss(LOSSES[loss], None if target is None else target.data_ptr(),
               None if weight is None else weight.data_ptr())
    _check(_lib.gs_grad_static(ctypes.byref(ps), ctypes.byref(ms), ctypes.byref(ls), _ptr(out.loss), _ptr(out.dp),
                               _ptr(out.du0), _ptr(out.dshared), _stream(stream)), "gs_grad_static")
    return out
