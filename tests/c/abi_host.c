/* A plain C99 client of libgradsolve: compiles against include/gradsolve.h
 * alone and exercises the host-side part of the ABI (status strings, workspace
 * sizing, argument validation, the no-op empty ensemble).  No call here
 * reaches the GPU: every request is either sized on the host or rejected, or
 * has n = 0, before anything would be launched.  Exit status 0 = all checks
 * held; otherwise the number of the first failed check. */
#include <stdio.h>
#include <string.h>

#include "gradsolve.h"

#define CHECK(id, cond)                               \
  do {                                                \
    if (!(cond)) {                                    \
      fprintf(stderr, "check %d failed: %s\n", id, #cond); \
      return id;                                      \
    }                                                 \
  } while (0)

int main(void) {
  const double tsave[2] = {0.5, 1.0};
  const int64_t before = gs_launch_count();
  gs_problem p;
  memset(&p, 0, sizeof p);
  p.system = GS_LORENZ;
  p.method = GS_TSIT5;
  p.dtype = GS_F64;
  p.d = 3;
  p.np = 3;
  p.n = 1000;
  p.p = (const void*)16; /* never dereferenced by the host-side calls below */
  p.u0 = (const void*)16;
  p.t0 = 0.0;
  p.t1 = 1.0;
  p.nsave = 2;
  p.tsave = tsave;
  gs_mesh m;
  memset(&m, 0, sizeof m);
  m.smax = 500;
  m.nsave = 2;
  gs_tol tol = {1e-6, 1e-6, 0.0, 0};

  /* status strings */
  CHECK(1, strcmp(gs_status_string(GS_OK), "ok") == 0);
  CHECK(2, strlen(gs_status_string(GS_EUNSUPPORTED)) > 0);
  /* workspace: one checkpointed state per step and slot, then (Tsit5 on
     Lorenz) the loss gradient of each save point */
  CHECK(3, gs_workspace_bytes(&p, &m, GS_OP_GRAD) == (size_t)(500 * 3 + 2 * 3) * 1000 * 8);
  p.dtype = GS_F32;
  CHECK(4, gs_workspace_bytes(&p, &m, GS_OP_GRAD) == (size_t)(500 * 3 + 2 * 3) * 1000 * 4);
  p.dtype = GS_F64;
  CHECK(5, gs_workspace_bytes(&p, &m, GS_OP_RECORD) >= (size_t)1000 * 4);
  /* kin8: d = np = 8, Rosenbrock only */
  p.system = GS_KIN8;
  p.method = GS_ROS3;
  p.d = p.np = 8;
  CHECK(6, gs_workspace_bytes(&p, &m, GS_OP_GRAD) == (size_t)500 * 8 * 1000 * 8);
  p.method = GS_TSIT5;
  CHECK(7, gs_count(&p, &tol, 100, (int32_t*)16, NULL, NULL) == GS_EUNSUPPORTED);
  p.method = GS_ROS2;
  p.d = p.np = 3;
  CHECK(8, gs_count(&p, &tol, 100, (int32_t*)16, NULL, NULL) == GS_EINVAL);
  /* HIRES is declared but not built */
  p.system = GS_HIRES;
  CHECK(9, gs_count(&p, &tol, 100, (int32_t*)16, NULL, NULL) == GS_EUNSUPPORTED);
  /* bad tolerances, save times out of range, too small a workspace */
  p.system = GS_LORENZ;
  p.method = GS_TSIT5;
  gs_tol bad = {-1.0, 1e-6, 0.0, 0};
  CHECK(10, gs_count(&p, &bad, 100, (int32_t*)16, NULL, NULL) == GS_EINVAL);
  const double late[1] = {2.0};
  p.tsave = late;
  p.nsave = 1;
  m.nsave = 1;
  CHECK(11, gs_count(&p, &tol, 100, (int32_t*)16, NULL, NULL) == GS_EINVAL);
  p.tsave = tsave;
  p.nsave = 2;
  m.nsave = 2;
  m.h = (void*)16;
  m.order = m.nsteps = m.save_idx = m.status = m.nreject = (int32_t*)16;
  CHECK(12, gs_record(&p, &tol, &m, (void*)16, 8, NULL) == GS_EWORKSPACE);
  gs_loss ls = {GS_LOSS_SUMSQ, NULL, NULL};
  CHECK(13, gs_grad(&p, &m, &ls, (void*)16, (void*)16, (void*)16, NULL, (void*)16, 8, NULL) == GS_EWORKSPACE);
  /* the in-place re-record and the ordered solve need their 8-byte counter */
  CHECK(17, gs_record_inplace(&p, &tol, &m, (void*)16, GS_RECORD_INPLACE_WS - 1, NULL) == GS_EWORKSPACE);
  CHECK(18, gs_record_inplace(&p, &tol, &m, (void*)20, GS_RECORD_INPLACE_WS, NULL) == GS_EINVAL);
  CHECK(19, gs_solve_adaptive_ordered(&p, &tol, 100, (const int32_t*)16, (void*)16, NULL, NULL, NULL, 0, NULL) ==
                GS_EWORKSPACE);
  CHECK(20, gs_solve_adaptive_ordered(&p, &tol, 100, NULL, (void*)16, NULL, NULL, (void*)16, 8, NULL) == GS_EINVAL);
  /* an empty ensemble is a no-op */
  p.n = 0;
  CHECK(14, gs_count(&p, &tol, 100, NULL, NULL, NULL) == GS_OK);
  CHECK(15, gs_grad(&p, &m, &ls, NULL, NULL, NULL, NULL, NULL, 0, NULL) == GS_OK);
  CHECK(21, gs_record_inplace(&p, &tol, &m, NULL, 0, NULL) == GS_OK);
  CHECK(16, gs_launch_count() == before);
  printf("ok\n");
  return 0;
}
