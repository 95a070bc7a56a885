// solve.cu -- forward-only fixed-step replay on a recorded mesh, writing the
// state at every save point (d = 3 systems with Tsit5, Verner 7, ROS2 or
// ROS3; the d = 8 system with ROS2 or ROS3).  The forward-only
// use of GRADSOLVE (arXiv 2609.02876, abstract); same arithmetic as the
// forward half of the gradient kernels.
#include "kin8.cuh"

namespace gs {

template <typename T>
struct SolveArgs {
  int64_t n;
  const T* p;
  const T* u0;
  const T* h;
  const int32_t* order;
  const int32_t* nsteps;
  const int32_t* save_idx;
  const int32_t* status;
  int32_t nsave;
  int32_t smax;
  const T* theta;  // [nsave][n] by slot: dense save points (d = 3 systems), or null
  T* u_save;       // [nsave][d][n] by trajectory
};

template <typename T, int SYS, int METHOD>
__global__ void __launch_bounds__(128) k_solve3(SolveArgs<T> a) {
  constexpr int D = SysDim<SYS>::D;
  const int64_t n = a.n;
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t i = a.order[j];
  if (i < 0 || i >= n) return;  // not a permutation entry: nothing to write
  const int64_t n3 = D * n;
  if (a.status[j] != GS_TRAJ_OK || a.nsteps[j] < 0 || a.nsteps[j] > a.smax) {
    const T nan = cst<T>(__longlong_as_double(0x7ff8000000000000ULL));
    for (int k = 0; k < a.nsave; ++k)
#pragma unroll
      for (int c = 0; c < D; ++c) a.u_save[k * n3 + c * n + i] = nan;
    return;
  }
  T u[D], p[D], k1[D];
#pragma unroll
  for (int c = 0; c < D; ++c) {
    u[c] = a.u0[c * n + i];
    p[c] = a.p[c * n + i];
  }
  rhs_s<T, SYS>(u, p, k1);
  const int S = a.nsteps[j];
  int kk = 0;
  int next = a.save_idx[j];
  const T* hp = a.h + j;
  for (int st = 0; st < S; ++st) {
    const T h = hp[(int64_t)st * n];
    T un[D];
    if constexpr (SYS == GS_KIN8) {
      T LU[64], R[8], q1[8], v[8], q2[8], q3[8];
      int P[8];
      if constexpr (METHOD == GS_ROS3)
        kin8_ros3_fwd<T>(u, p, h, LU, P, R, q1, v, q2, q3, un);
      else
        kin8_ros2_fwd<T>(u, p, h, LU, P, R, q1, v, q2, un);
    } else if constexpr (METHOD == GS_VERN7) {
      vern7_step3<T, SYS>(u, p, h, k1, un, nullptr);
      rhs3<T, SYS>(un, p, k1);  // the next step's first slope (not FSAL)
    } else if constexpr (METHOD == GS_TSIT5) {
      T k7[3], e[3];
      tsit5_err_step<T, SYS>(u, p, h, k1, un, k7, e);
      if (a.theta) {
        // dense save points inside this step: Tsit5's continuous extension
        // over the step's stages, recomputed from u and k1
        while (st + 1 == next) {
          const T th = a.theta[(int64_t)kk * n + j];
          T ut[3] = {un[0], un[1], un[2]};
          if (th != cst<T>(1.0)) tsit5_dense3<T, SYS>(u, p, h, k1, th, ut);
#pragma unroll
          for (int c = 0; c < 3; ++c) a.u_save[kk * n3 + c * n + i] = ut[c];
          ++kk;
          next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
        }
      }
#pragma unroll
      for (int c = 0; c < 3; ++c) k1[c] = k7[c];
    } else {
      T LU[9], R[3], q1[3], v[3], q2[3];
      int P[3];
      if constexpr (METHOD == GS_ROS3) {
        T q3[3];
        ros3_fwd<T, SYS>(u, p, h, LU, P, R, q1, v, q2, q3, un);
      } else {
        ros2_fwd<T, SYS>(u, p, h, LU, P, R, q1, v, q2, un);
      }
      if (a.theta && st + 1 == next) {
        // dense save points inside this step: the Hermite state on u, f(u),
        // u_new, f(u_new), the slopes evaluated here
        T fs[3], fn[3];
        rhs3<T, SYS>(u, p, fs);
        rhs3<T, SYS>(un, p, fn);
        while (st + 1 == next) {
          const T th = a.theta[(int64_t)kk * n + j];
          const HermiteW<T> w = hermite_w(th);
#pragma unroll
          for (int c = 0; c < 3; ++c)
            a.u_save[kk * n3 + c * n + i] = th == cst<T>(1.0) ? un[c] : hermite_c(w, u[c], un[c], fs[c], fn[c], h);
          ++kk;
          next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
        }
      }
    }
#pragma unroll
    for (int c = 0; c < D; ++c) u[c] = un[c];
    while (st + 1 == next) {
#pragma unroll
      for (int c = 0; c < D; ++c) a.u_save[kk * n3 + c * n + i] = u[c];
      ++kk;
      next = kk < a.nsave ? a.save_idx[(int64_t)kk * n + j] : -1;
    }
  }
}

template <typename T>
gs_status launch_solve3(const gs_problem* P, const gs_mesh* M, void* u_save, cudaStream_t st) {
  SolveArgs<T> a;
  a.n = P->n;
  a.p = (const T*)P->p;
  a.u0 = (const T*)P->u0;
  a.h = (const T*)M->h;
  a.order = M->order;
  a.nsteps = M->nsteps;
  a.save_idx = M->save_idx;
  a.status = M->status;
  a.nsave = P->nsave;
  a.smax = M->smax;
  a.theta = P->system != GS_KIN8 ? (const T*)M->save_theta : nullptr;
  a.u_save = (T*)u_save;
  const unsigned grid = (unsigned)((P->n + 127) / 128);
  if (P->system == GS_LORENZ && P->method == GS_TSIT5)
    k_solve3<T, kSysLorenz, GS_TSIT5><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_LORENZ && P->method == GS_ROS2)
    k_solve3<T, kSysLorenz, GS_ROS2><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_LORENZ && P->method == GS_ROS3)
    k_solve3<T, kSysLorenz, GS_ROS3><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_ROBERTSON && P->method == GS_TSIT5)
    k_solve3<T, kSysRobertson, GS_TSIT5><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_ROBERTSON && P->method == GS_ROS3)
    k_solve3<T, kSysRobertson, GS_ROS3><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_KIN8 && P->method == GS_ROS3)
    k_solve3<T, kSysKin8, GS_ROS3><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_KIN8 && P->method == GS_ROS2)
    k_solve3<T, kSysKin8, GS_ROS2><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_LORENZ && P->method == GS_VERN7)
    k_solve3<T, kSysLorenz, GS_VERN7><<<grid, 128, 0, st>>>(a);
  else if (P->system == GS_ROBERTSON && P->method == GS_VERN7)
    k_solve3<T, kSysRobertson, GS_VERN7><<<grid, 128, 0, st>>>(a);
  else
    k_solve3<T, kSysRobertson, GS_ROS2><<<grid, 128, 0, st>>>(a);
  count_launch();
  return launch_ok() ? GS_OK : GS_ECUDA;
}

template gs_status launch_solve3<double>(const gs_problem*, const gs_mesh*, void*, cudaStream_t);
template gs_status launch_solve3<float>(const gs_problem*, const gs_mesh*, void*, cudaStream_t);

}  // namespace gs
