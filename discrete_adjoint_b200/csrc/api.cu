// api.cu -- the C ABI of libgradsolve: argument validation, workspace sizing
// and dispatch to the kernels.  Nothing here allocates device memory; every
// device buffer is the caller's (see include/gradsolve.h).
#include <atomic>
#include <cmath>

#include "common.cuh"

namespace gs {

static std::atomic<int64_t> g_launches{0};
void count_launch(int k) { g_launches.fetch_add(k, std::memory_order_relaxed); }

// kernels (defined in the other translation units)
gs_status count3(const gs_problem*, const gs_tol*, int32_t, int32_t*, int32_t*, cudaStream_t);
gs_status record3(const gs_problem*, const gs_tol*, const gs_mesh*, void*, cudaStream_t);
gs_status record3_inplace(const gs_problem*, const gs_tol*, const gs_mesh*, void*, cudaStream_t);
gs_status solve_adaptive3(const gs_problem*, const gs_tol*, int32_t, void*, int32_t*, int32_t*, cudaStream_t);
gs_status solve_adaptive3_ordered(const gs_problem*, const gs_tol*, int32_t, const int32_t*, void*, int32_t*,
                                  int32_t*, void*, cudaStream_t);
size_t record_ws_bytes(int64_t n, int32_t smax, int32_t nsave, size_t tsize);
template <typename T>
gs_status launch_grad_tsit5_lorenz(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                                   cudaStream_t);
template <typename T>
gs_status launch_sens_tsit5_lorenz(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                                   cudaStream_t);
template <typename T>
gs_status launch_sens_ros(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                          cudaStream_t);
template <typename T>
gs_status launch_sens_vern7_lorenz(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                                   cudaStream_t);
template <typename T>
gs_status launch_sens_kin8(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                           cudaStream_t);
template <typename T>
gs_status launch_grad_ros2(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                           cudaStream_t);
template <typename T>
gs_status launch_grad_ros3(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                           cudaStream_t);
template <typename T>
gs_status launch_grad_kin8(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                           cudaStream_t);
template <typename T>
gs_status launch_grad_vern7_lorenz(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*,
                                   cudaStream_t);
template <typename T>
gs_status launch_solve3(const gs_problem*, const gs_mesh*, void*, cudaStream_t);
gs_status record_node64(const gs_problem*, const gs_tol*, const gs_mesh*, void*, cudaStream_t);
gs_status node64_record_pass(const gs_problem*, const gs_tol*, int32_t, bool, float*, int32_t*, int32_t*, int32_t*,
                             int32_t*, cudaStream_t, float*);
gs_status node64_grad(const gs_problem*, const gs_mesh*, const gs_loss*, void*, void*, void*, void*, void*,
                      cudaStream_t);
gs_status node64_solve(const gs_problem*, const gs_mesh*, void*, cudaStream_t);
void node64_set_tensor(int on);
size_t node64_grad_ws_bytes(int64_t n, int32_t smax, size_t tsize);
size_t grad_tsit5_lorenz_ws_bytes(int32_t dtype, int64_t n, int32_t smax, int32_t nsave, bool dense);
size_t grad_vern7_lorenz_ws_bytes(int32_t dtype, int64_t n, int32_t smax, int32_t nsave);

static size_t dsize(const gs_problem* P) { return P->dtype == GS_F64 ? 8 : 4; }

static gs_status check_problem(const gs_problem* P) {
  if (!P) return GS_EINVAL;
  if (P->n < 0 || P->n > (int64_t)INT32_MAX) return GS_EINVAL;
  if (P->dtype != GS_F32 && P->dtype != GS_F64) return GS_EINVAL;
  if (P->method != GS_TSIT5 && P->method != GS_ROS2 && P->method != GS_ROS3 && P->method != GS_VERN7)
    return GS_EINVAL;
  switch (P->system) {
    case GS_LORENZ:
    case GS_ROBERTSON:
      if (P->d != 3 || P->np != 3) return GS_EINVAL;
      break;
    case GS_NODE64:
      if (P->d != 64 || P->np != 64) return GS_EINVAL;
      if (P->n > 0 && !P->shared) return GS_EINVAL;
      // built for the single-precision Tsit5 configuration
      if (P->method != GS_TSIT5 || P->dtype != GS_F32) return GS_EUNSUPPORTED;
      break;
    case GS_KIN8:
      if (P->d != 8 || P->np != 8) return GS_EINVAL;
      // a stiff system: built for the Rosenbrock methods
      if (P->method == GS_TSIT5 || P->method == GS_VERN7) return GS_EUNSUPPORTED;
      break;
    case GS_HIRES:
      return GS_EUNSUPPORTED;
    default:
      return GS_EINVAL;
  }
  if (P->n > 0 && (!P->p || !P->u0)) return GS_EINVAL;
  if (!std::isfinite(P->t0) || !std::isfinite(P->t1) || !(P->t0 < P->t1)) return GS_EINVAL;
  if (P->nsave < 1 || P->nsave > GS_MAX_SAVE || !P->tsave) return GS_EINVAL;
  double prev = P->t0;
  for (int k = 0; k < P->nsave; ++k) {
    const double t = P->tsave[k];
    if (!(t > prev) || !(t <= P->t1)) return GS_EINVAL;
    prev = t;
  }
  return GS_OK;
}

static gs_status check_mesh(const gs_problem* P, const gs_mesh* M) {
  if (!M) return GS_EINVAL;
  if (M->smax < 1 || M->nsave != P->nsave) return GS_EINVAL;
  if (P->n > 0 && (!M->h || !M->order || !M->nsteps || !M->save_idx || !M->status)) return GS_EINVAL;
  return GS_OK;
}

// Tolerances; a dense record is built for the d = 3 systems (Tsit5, ROS2 and
// ROS3; Verner's pair has landing records only).
static gs_status check_tol(const gs_problem* P, const gs_tol* tol) {
  if (!tol || !(tol->rtol >= 0) || !(tol->atol >= 0) || !(tol->rtol + tol->atol > 0) || !(tol->h0 >= 0))
    return GS_EINVAL;
  if (tol->dense != 0 && tol->dense != 1) return GS_EINVAL;
  if (tol->dense && (P->system == GS_NODE64 || P->system == GS_KIN8 || P->method == GS_VERN7))
    return GS_EUNSUPPORTED;
  return GS_OK;
}

}  // namespace gs

using namespace gs;

extern "C" {

gs_status gs_set_option(int32_t option, int32_t value) {
  if (option == GS_OPT_NODE64_TENSOR_CORES && (value == 0 || value == 1)) {
    node64_set_tensor(value);
    return GS_OK;
  }
  return GS_EINVAL;
}

const char* gs_status_string(gs_status s) {
  switch (s) {
    case GS_OK: return "ok";
    case GS_EINVAL: return "invalid argument";
    case GS_ECUDA: return "CUDA error";
    case GS_EWORKSPACE: return "workspace missing or too small";
    case GS_EUNSUPPORTED: return "unsupported system/method/dtype combination";
    default: return "unknown status";
  }
}

int64_t gs_launch_count(void) { return g_launches.load(); }

size_t gs_workspace_bytes(const gs_problem* P, const gs_mesh* M, int32_t op) {
  if (check_problem(P) != GS_OK || !M || M->smax < 1) return 0;
  if (op == GS_OP_RECORD) return record_ws_bytes(P->n, M->smax, P->nsave, dsize(P));
  if (op == GS_OP_GRAD) {
    if (P->system == GS_NODE64) return node64_grad_ws_bytes(P->n, M->smax, dsize(P));
    // one checkpointed state per step and slot (the Tsit5 and Verner Lorenz
    // kernels add the save points' loss gradients)
    if (P->method == GS_TSIT5 && P->system == GS_LORENZ)
      return grad_tsit5_lorenz_ws_bytes(P->dtype, P->n, M->smax, P->nsave, M->save_theta != nullptr);
    if (P->method == GS_VERN7 && P->system == GS_LORENZ)
      return grad_vern7_lorenz_ws_bytes(P->dtype, P->n, M->smax, P->nsave);
    return (size_t)M->smax * (size_t)P->d * (size_t)P->n * dsize(P);
  }
  return 0;
}

gs_status gs_count(const gs_problem* P, const gs_tol* tol, int32_t smax, int32_t* nsteps, int32_t* status,
                   void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_tol(P, tol)) != GS_OK) return rc;
  if (smax < 1) return GS_EINVAL;
  if (P->n == 0) return GS_OK;
  if (!nsteps) return GS_EINVAL;
  if (P->system == GS_NODE64)
    return node64_record_pass(P, tol, smax, false, nullptr, nullptr, nsteps, status, nullptr, (cudaStream_t)stream,
                              nullptr);
  return count3(P, tol, smax, nsteps, status, (cudaStream_t)stream);
}

gs_status gs_solve_adaptive(const gs_problem* P, const gs_tol* tol, int32_t smax, void* u_save, int32_t* nsteps,
                            int32_t* status, void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_tol(P, tol)) != GS_OK) return rc;
  if (smax < 1) return GS_EINVAL;
  if (P->n == 0) return GS_OK;
  if (!u_save) return GS_EINVAL;
  if (P->system == GS_NODE64)
    return node64_record_pass(P, tol, smax, false, nullptr, nullptr, nsteps, status, nullptr, (cudaStream_t)stream,
                              (float*)u_save);
  return solve_adaptive3(P, tol, smax, u_save, nsteps, status, (cudaStream_t)stream);
}

gs_status gs_record(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, size_t ws_bytes,
                    void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_mesh(P, M)) != GS_OK) return rc;
  if ((rc = check_tol(P, tol)) != GS_OK) return rc;
  if (tol->dense && P->n > 0 && !M->save_theta) return GS_EINVAL;  // a dense record writes the positions
  if (P->n == 0) return GS_OK;
  if (!ws || ws_bytes < gs_workspace_bytes(P, M, GS_OP_RECORD)) return GS_EWORKSPACE;
  if (P->system == GS_NODE64) return record_node64(P, tol, M, ws, (cudaStream_t)stream);
  return record3(P, tol, M, ws, (cudaStream_t)stream);
}

gs_status gs_solve_adaptive_ordered(const gs_problem* P, const gs_tol* tol, int32_t smax, const int32_t* order,
                                    void* u_save, int32_t* nsteps, int32_t* status, void* ws, size_t ws_bytes,
                                    void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_tol(P, tol)) != GS_OK) return rc;
  if (smax < 1) return GS_EINVAL;
  if (P->system == GS_NODE64) return GS_EUNSUPPORTED;
  if (P->n == 0) return GS_OK;
  if (!u_save || !order) return GS_EINVAL;
  if (!ws || ws_bytes < GS_RECORD_INPLACE_WS) return GS_EWORKSPACE;
  if ((uintptr_t)ws % 8 != 0) return GS_EINVAL;
  return solve_adaptive3_ordered(P, tol, smax, order, u_save, nsteps, status, ws, (cudaStream_t)stream);
}

gs_status gs_record_inplace(const gs_problem* P, const gs_tol* tol, const gs_mesh* M, void* ws, size_t ws_bytes,
                            void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_mesh(P, M)) != GS_OK) return rc;
  if ((rc = check_tol(P, tol)) != GS_OK) return rc;
  if (P->system == GS_NODE64) return GS_EUNSUPPORTED;
  if (tol->dense && P->n > 0 && !M->save_theta) return GS_EINVAL;  // a dense record writes the positions
  if (P->n == 0) return GS_OK;
  if (!ws || ws_bytes < GS_RECORD_INPLACE_WS) return GS_EWORKSPACE;
  if ((uintptr_t)ws % 8 != 0) return GS_EINVAL;
  return record3_inplace(P, tol, M, ws, (cudaStream_t)stream);
}

gs_status gs_solve(const gs_problem* P, const gs_mesh* M, void* u_save, void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_mesh(P, M)) != GS_OK) return rc;
  if (M->save_theta && (P->system == GS_NODE64 || P->system == GS_KIN8 || P->method == GS_VERN7))
    return GS_EUNSUPPORTED;
  if (P->n == 0) return GS_OK;
  if (!u_save) return GS_EINVAL;
  if (P->system == GS_NODE64) return node64_solve(P, M, u_save, (cudaStream_t)stream);
  return P->dtype == GS_F64 ? launch_solve3<double>(P, M, u_save, (cudaStream_t)stream)
                            : launch_solve3<float>(P, M, u_save, (cudaStream_t)stream);
}

gs_status gs_grad(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                  void* dshared, void* ws, size_t ws_bytes, void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_mesh(P, M)) != GS_OK) return rc;
  if (!Ls || (Ls->kind != GS_LOSS_SUMSQ && Ls->kind != GS_LOSS_LINEAR)) return GS_EINVAL;
  // dense save points: the d = 3 gradients (Tsit5 on Lorenz, ROS2 / ROS3 on Lorenz and Robertson)
  if (M->save_theta && (P->system == GS_NODE64 || P->system == GS_KIN8 || P->method == GS_VERN7))
    return GS_EUNSUPPORTED;
  // Verner's pair: the Lorenz gradient
  if (P->method == GS_VERN7 && P->system != GS_LORENZ) return GS_EUNSUPPORTED;
  if (P->n == 0) return GS_OK;
  if (Ls->kind == GS_LOSS_LINEAR && !Ls->weight) return GS_EINVAL;
  if (!loss || !dp || !du0) return GS_EINVAL;
  if (!ws || ws_bytes < gs_workspace_bytes(P, M, GS_OP_GRAD)) return GS_EWORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  if (P->system == GS_NODE64) return node64_grad(P, M, Ls, loss, dp, du0, dshared, ws, st);
  if (P->method == GS_TSIT5 && P->system == GS_LORENZ)
    return P->dtype == GS_F64 ? launch_grad_tsit5_lorenz<double>(P, M, Ls, loss, dp, du0, ws, st)
                              : launch_grad_tsit5_lorenz<float>(P, M, Ls, loss, dp, du0, ws, st);
  if (P->method == GS_VERN7)
    return P->dtype == GS_F64 ? launch_grad_vern7_lorenz<double>(P, M, Ls, loss, dp, du0, ws, st)
                              : launch_grad_vern7_lorenz<float>(P, M, Ls, loss, dp, du0, ws, st);
  if (P->system == GS_KIN8)
    return P->dtype == GS_F64 ? launch_grad_kin8<double>(P, M, Ls, loss, dp, du0, ws, st)
                              : launch_grad_kin8<float>(P, M, Ls, loss, dp, du0, ws, st);
  if (P->method == GS_ROS2)
    return P->dtype == GS_F64 ? launch_grad_ros2<double>(P, M, Ls, loss, dp, du0, ws, st)
                              : launch_grad_ros2<float>(P, M, Ls, loss, dp, du0, ws, st);
  if (P->method == GS_ROS3)
    return P->dtype == GS_F64 ? launch_grad_ros3<double>(P, M, Ls, loss, dp, du0, ws, st)
                              : launch_grad_ros3<float>(P, M, Ls, loss, dp, du0, ws, st);
  return GS_EUNSUPPORTED;
}

gs_status gs_sens(const gs_problem* P, const gs_mesh* M, const gs_loss* Ls, void* loss, void* dp, void* du0,
                  void* sens, void* stream) {
  gs_status rc = check_problem(P);
  if (rc != GS_OK) return rc;
  if ((rc = check_mesh(P, M)) != GS_OK) return rc;
  if (!Ls || (Ls->kind != GS_LOSS_SUMSQ && Ls->kind != GS_LOSS_LINEAR)) return GS_EINVAL;
  // Tsit5: Lorenz; ROS2 / ROS3: Lorenz and Robertson (landing or dense save
  // points) and kin8 (landing)
  if (P->system == GS_NODE64) return GS_EUNSUPPORTED;
  if (P->system == GS_KIN8 && M->save_theta) return GS_EUNSUPPORTED;
  // Verner's pair: Lorenz, landing meshes
  if (P->method == GS_VERN7 && (P->system != GS_LORENZ || M->save_theta)) return GS_EUNSUPPORTED;
  if (P->method == GS_TSIT5 && P->system != GS_LORENZ) return GS_EUNSUPPORTED;
  if (P->n == 0) return GS_OK;
  if (Ls->kind == GS_LOSS_LINEAR && !Ls->weight) return GS_EINVAL;
  if (!loss || !dp || !du0) return GS_EINVAL;
  cudaStream_t st = (cudaStream_t)stream;
  if (P->system == GS_KIN8)
    return P->dtype == GS_F64 ? launch_sens_kin8<double>(P, M, Ls, loss, dp, du0, sens, st)
                              : launch_sens_kin8<float>(P, M, Ls, loss, dp, du0, sens, st);
  if (P->method == GS_VERN7)
    return P->dtype == GS_F64 ? launch_sens_vern7_lorenz<double>(P, M, Ls, loss, dp, du0, sens, st)
                              : launch_sens_vern7_lorenz<float>(P, M, Ls, loss, dp, du0, sens, st);
  if (P->method != GS_TSIT5)
    return P->dtype == GS_F64 ? launch_sens_ros<double>(P, M, Ls, loss, dp, du0, sens, st)
                              : launch_sens_ros<float>(P, M, Ls, loss, dp, du0, sens, st);
  return P->dtype == GS_F64 ? launch_sens_tsit5_lorenz<double>(P, M, Ls, loss, dp, du0, sens, st)
                            : launch_sens_tsit5_lorenz<float>(P, M, Ls, loss, dp, du0, sens, st);
}

}  // extern "C"
