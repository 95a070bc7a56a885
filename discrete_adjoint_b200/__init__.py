"""B200 record-and-replay discrete adjoints for ODE ensembles.

The compute path is libgradsolve.so (hand-written CUDA for sm_100a, C ABI in
include/gradsolve.h); ``gradsolve`` is its thin ctypes binding.  Importing the
package loads the library and fails if it has not been built.
"""
from . import gradsolve
from .gradsolve import (Ensemble, GradOut, Mesh, gs_count, gs_grad, gs_grad_static, gs_launch_count, gs_record,
                        gs_record_inplace, gs_sens, gs_set_option, gs_solve, gs_solve_adaptive,
                        gs_solve_adaptive_ordered, gs_status_string, gs_workspace_bytes, new_grad_out, new_mesh,
                        workspace)

__all__ = ["gradsolve", "Ensemble", "GradOut", "Mesh", "gs_count", "gs_grad", "gs_grad_static", "gs_launch_count",
           "gs_record", "gs_record_inplace", "gs_sens", "gs_set_option", "gs_solve", "gs_solve_adaptive",
           "gs_solve_adaptive_ordered", "gs_status_string", "gs_workspace_bytes", "new_grad_out", "new_mesh",
           "workspace"]
